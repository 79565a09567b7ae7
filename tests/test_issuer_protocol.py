"""Model check of the band kernel's barrier protocol (host only, no GPU).

The persistent band kernel runs one TMA producer, one or two MMA issuers and two
softmax groups that hand work to each other through mbarriers (csrc/band_tc.cu).
This test replays that protocol as a discrete-event simulation with a random
scheduler over random unit shapes, for both TMEM layouts:

* P over S (D = 128): one issuer for both query tiles, P published in two halves,
  the next S issued after the PV that reads P;
* separate P (D = 64): one issuer per query tile, the next S issued as soon as the
  softmax has read the current one (up to NS - 1 key tiles ahead), and every
  issuer releasing every K/V ring slot of the unit (kv_empty counts two arrivals).

MMAs complete asynchronously and in issue order per issuer; a commit arrives on its
barrier once the MMAs issued before it have completed.  Checked on every run:

* no deadlock: every agent finishes;
* no parity-ambiguous wait: a barrier is never two phases ahead of a waiter (the
  hardware's parity test would then block for good);
* no K/V slot is refilled while an MMA that reads its previous contents is pending;
* every query tile's softmax sees exactly its own key tiles, in order.

Optionally both softmax groups also meet at every unit start, as they do when a side
or local bias is staged in shared memory.  Two more models cover the backward
(csrc/bwd_tc.cu): the key-stationary dK/dV pass and the pipelined query-stationary dQ
pass.  Each model has a planted-mistake test.
"""
import random

import pytest


class Barrier:
    def __init__(self, name, count):
        self.name, self.count, self.arrivals, self.done = name, count, 0, 0

    def arrive(self):
        self.arrivals += 1
        assert self.arrivals <= self.count
        if self.arrivals == self.count:
            self.arrivals = 0
            self.done += 1


class ProtocolError(AssertionError):
    pass


def wait(bar, k):
    """Generator step: wait for the completion of phase k (parity wait)."""
    while True:
        if bar.done - k >= 2:
            raise ProtocolError(f"{bar.name}: {bar.done} phases done, waiter on phase {k}")
        if bar.done > k:
            return
        yield


def random_units(rng, n_units):
    """Tile lists of random units, shaped as the kernel builds them: band tiles from
    the first key of tile A's window, so A uses tiles 0..a_hi and B, whose rows start
    128 class rows later, tiles b_lo..nband-1 with b_lo 0 (paired heads or a window
    reaching back a whole tile) or 1; the band is the union of the two windows; then
    global and side tiles (both tiles), then the random tiles, alternating A, B."""
    units = []
    for _ in range(n_units):
        kind = rng.random()
        nband = rng.randint(1, 5)
        b_active = rng.random() > 0.15
        if b_active:
            b_lo = rng.randint(0, min(1, nband - 1))
            a_hi = rng.randint(max(0, b_lo - 1), nband - 1)
        else:
            b_lo, a_hi = nband, nband - 1
        use_a = [j <= a_hi for j in range(nband)]
        use_b = [b_active and j >= b_lo for j in range(nband)]
        extra = rng.randint(0, 3) if kind < 0.5 else 0        # global / side tiles: both tiles
        use_a += [True] * extra
        use_b += [b_active] * extra
        nr = rng.randint(0, 3) if kind > 0.7 else 0           # random tiles, alternating
        for t in range(nr):
            for x in range(2 if b_active else 1):
                use_a.append(x == 0)
                use_b.append(x == 1)
        units.append((use_a, use_b, b_active))
    return units


def simulate(seed, sep_p, staged=False, n_units=12):
    rng = random.Random(seed)
    NS = 4 if sep_p else 2
    issuers = 2 if sep_p else 1
    units = random_units(rng, n_units)
    B = {}

    def bar(name, count=1):
        B[name] = Barrier(name, count)
        return B[name]

    q_full = [bar(f"q_full{x}") for x in range(2)]
    q_empty = [bar(f"q_empty{x}") for x in range(2)]
    k_full = [bar(f"k_full{s}") for s in range(NS)]
    v_full = [bar(f"v_full{s}") for s in range(NS)]
    kv_empty = [bar(f"kv_empty{s}", issuers) for s in range(NS)]
    s_full = [bar(f"s_full{x}") for x in range(2)]
    s_free = [bar(f"s_free{x}", 128) for x in range(2)]
    p_half = [bar(f"p_half{x}", 128) for x in range(2)]
    p_full = [bar(f"p_full{x}", 128) for x in range(2)]
    pv_done = [bar(f"pv_done{x}") for x in range(2)]
    o_full = [bar(f"o_full{x}") for x in range(2)]

    # per issuer: FIFO of ('mma', (slot, use)) and ('commit', barrier) entries
    pipes = [[] for _ in range(issuers)]
    pending_reads = {}                       # (slot, use) -> MMAs not yet complete
    loads = [0] * NS                         # loads into each slot so far
    seen = [[], []]                          # key tiles each softmax group processed

    def mma(i, slot):
        key = (slot, loads[slot] - 1)
        pending_reads[key] = pending_reads.get(key, 0) + 1
        pipes[i].append(("mma", key))

    def commit(i, b):
        pipes[i].append(("commit", b))

    def producer():
        qloads = [0, 0]
        kv = 0
        for use_a, use_b, b_act in units:
            for x, act in ((0, True), (1, b_act)):
                if not act:
                    continue
                if qloads[x] > 0:
                    yield from wait(q_empty[x], qloads[x] - 1)
                q_full[x].arrive()
                qloads[x] += 1
            for j in range(len(use_a)):
                st = kv % NS
                if kv >= NS:
                    yield from wait(kv_empty[st], kv // NS - 1)
                if pending_reads.get((st, loads[st] - 1), 0):
                    raise ProtocolError(f"slot {st} refilled while an MMA still reads it")
                loads[st] += 1
                yield
                k_full[st].arrive()
                yield
                v_full[st].arrive()
                kv += 1

    def issuer(i):
        xs = [i] if issuers == 2 else [0, 1]
        qwaits = {x: 0 for x in xs}
        pwaits = {x: 0 for x in xs}
        nqk = {x: 0 for x in xs}
        kv = 0
        for use_a, use_b, b_act in units:
            use = {0: use_a, 1: use_b}
            T = len(use_a)
            act = {x: (x == 0 or b_act) for x in xs}
            first = {x: next((j for j in range(T) if use[x][j]), -1) for x in xs}
            last = {x: max((j for j in range(T) if use[x][j]), default=-1) for x in xs}
            issued = {x: -1 for x in xs}

            def issue_qk(x, j):
                g = kv + j
                yield from wait(k_full[g % NS], g // NS)
                if sep_p and nqk[x] > 0:
                    yield from wait(s_free[x], nqk[x] - 1)
                nqk[x] += 1
                mma(i, g % NS)
                commit(i, s_full[x])
                if j == last[x]:
                    commit(i, q_empty[x])
                issued[x] = j

            for x in xs:
                if act[x] and first[x] >= 0:
                    yield from wait(q_full[x], qwaits[x])
                    qwaits[x] += 1
                    yield from issue_qk(x, first[x])
            for j in range(T):
                g = kv + j
                st = g % NS
                anyuse = False
                for x in xs:
                    u = act[x] and use[x][j]
                    anyuse = anyuse or u
                    if u and issued[x] < j:
                        yield from issue_qk(x, j)
                if sep_p:
                    for x in xs:
                        if not (act[x] and use[x][j]) or issued[x] != j:
                            continue
                        jn = j + 1
                        while jn < T and jn < j + NS and not use[x][jn]:
                            jn += 1
                        if jn < T and jn < j + NS:
                            yield from issue_qk(x, jn)
                yield from wait(v_full[st], g // NS)
                if not anyuse:
                    kv_empty[st].arrive()
                    continue
                for x in xs:
                    if not (act[x] and use[x][j]):
                        continue
                    if not sep_p:
                        yield from wait(p_half[x], pwaits[x])
                        mma(i, st)
                    yield from wait(p_full[x], pwaits[x])
                    pwaits[x] += 1
                    mma(i, st)
                    if sep_p:
                        commit(i, pv_done[x])
                    if j == last[x]:
                        commit(i, o_full[x])
                    elif not sep_p and j + 1 < T and use[x][j + 1]:
                        yield from issue_qk(x, j + 1)
                commit(i, kv_empty[st])
            kv += T

    met = {}                                 # unit -> softmax groups at the staging barrier

    def softmax(x):
        it = pw = oc = 0
        for u, (use_a, use_b, b_act) in enumerate(units):
            if staged:
                # a side or local bias is staged per unit by both groups together
                # (a named barrier over both groups, also when tile B is inactive)
                met[u] = met.get(u, 0) + 1
                while met[u] < 2:
                    yield
            if x == 1 and not b_act:
                continue
            use = use_a if x == 0 else use_b
            for j in range(len(use)):
                if not use[j]:
                    continue
                yield from wait(s_full[x], it)
                seen[x].append(j)
                if sep_p:
                    for _ in range(128):
                        s_free[x].arrive()
                yield
                if sep_p and pw > 0:
                    yield from wait(pv_done[x], pw - 1)
                if not sep_p:
                    for _ in range(128):
                        p_half[x].arrive()
                    yield
                for _ in range(128):
                    p_full[x].arrive()
                pw += 1
                it += 1
            yield from wait(o_full[x], oc)
            oc += 1

    agents = [producer()] + [issuer(i) for i in range(issuers)] + [softmax(0), softmax(1)]
    alive = list(range(len(agents)))

    def step_pipe(i):
        kind, val = pipes[i].pop(0)
        if kind == "mma":
            pending_reads[val] -= 1
        else:
            val.arrive()

    stalls = 0
    while alive or any(pipes):
        choices = [("agent", a) for a in alive] + [("pipe", i) for i in range(issuers) if pipes[i]]
        kind, who = rng.choice(choices)
        if kind == "pipe":
            step_pipe(who)
            stalls = 0
            continue
        try:
            next(agents[who])
            stalls += 1
        except StopIteration:
            alive.remove(who)
            stalls = 0
        if stalls > 20000:
            raise ProtocolError("deadlock: no agent can make progress")

    for x in range(2):
        expect = []
        for use_a, use_b, b_act in units:
            if x == 1 and not b_act:
                continue
            expect += [j for j, u in enumerate(use_a if x == 0 else use_b) if u]
        assert seen[x] == expect


@pytest.mark.parametrize("staged", [False, True], ids=["", "bias_staged"])
@pytest.mark.parametrize("sep_p", [False, True], ids=["p_over_s_one_issuer", "separate_p_two_issuers"])
def test_barrier_protocol_random_schedules(sep_p, staged):
    for seed in range(300):
        simulate(seed, sep_p, staged)


def test_model_detects_a_broken_release_count():
    """The model is not vacuous: with kv_empty counting one arrival while two
    issuers release every slot, a slot gets refilled under a pending reader or a
    barrier runs two phases ahead of a waiter on some schedule."""
    orig = Barrier.__init__

    def one_arrival(self, name, count):
        orig(self, name, 1 if name.startswith("kv_empty") else count)

    Barrier.__init__ = one_arrival
    try:
        caught = 0
        for seed in range(300):
            try:
                simulate(seed, True)
            except AssertionError:
                caught += 1
        assert caught > 0
    finally:
        Barrier.__init__ = orig


def simulate_dkv(seed, T, early_next=False, NR=4):
    """The key-stationary dK/dV pass (csrc/bwd_tc.cu): one key tile per CTA, its T
    query tiles through an NR-stage ring, compute groups taking alternate tiles.  A
    group writes Pᵀ and dSᵀ as bf16 over the TMEM columns of its Sᵀ and dPᵀ, and the
    dV / dK products read them from there; the group's next Sᵀ/dPᵀ is issued once
    those products are issued, so the in-order tensor pipe writes the columns only
    after the products have read them."""
    rng = random.Random(seed)
    a_full = Barrier("a_full", 1)
    r_full = [Barrier(f"r_full{s}", 1) for s in range(NR)]
    r_empty = [Barrier(f"r_empty{s}", 1) for s in range(NR)]
    s_full = [Barrier(f"s_full{g}", 1) for g in range(2)]
    p_full = [Barrier(f"p_full{g}", 128) for g in range(2)]
    acc_full = Barrier("acc_full", 1)
    pipe = []
    pending = {}
    loads = [0] * NR
    tm_uses = [0, 0]                        # P^T / dS^T written into each group's columns
    consumed = [0, 0]                       # tiles whose S^T/dP^T each group has read

    def mma(key):
        pending[key] = pending.get(key, 0) + 1
        pipe.append(("mma", key))

    def producer():
        a_full.arrive()
        for j in range(T):
            st = j % NR
            if j >= NR:
                yield from wait(r_empty[st], j // NR - 1)
            if pending.get(("ring", st, loads[st] - 1), 0):
                raise ProtocolError(f"ring slot {st} refilled under a pending reader")
            loads[st] += 1
            yield
            r_full[st].arrive()

    def issuer():
        def issue_s(j):
            st, g = j % NR, j & 1
            yield from wait(r_full[st], j // NR)
            if consumed[g] < (j >> 1):
                raise ProtocolError(f"S^T of tile {j} written before group {g} read tile {j - 2}")
            mma(("ring", st, loads[st] - 1))
            pipe.append(("write_tm", g))       # S^T / dP^T land in the group's columns
            pipe.append(("commit", s_full[g]))

        yield from wait(a_full, 0)
        yield from issue_s(0)
        if T > 1:
            yield from issue_s(1)
        for j in range(T):
            g, st = j & 1, j % NR
            if early_next and j + 2 < T:         # planted mistake: before the group read S(j)
                yield from issue_s(j + 2)
            yield from wait(p_full[g], j >> 1)
            mma(("ring", st, loads[st] - 1))
            mma(("tm", g, tm_uses[g] - 1))       # dV, dK read P^T, dS^T from TMEM
            pipe.append(("commit", r_empty[st]))
            if j + 2 < T and not early_next:
                yield from issue_s(j + 2)
        pipe.append(("commit", acc_full))

    def compute(g):
        nt = 0
        for j in range(g, T, 2):
            yield from wait(s_full[g], nt)
            consumed[g] += 1
            if pending.get(("tm", g, tm_uses[g] - 1), 0):
                raise ProtocolError(f"P^T of group {g} rewritten under a pending product")
            tm_uses[g] += 1
            yield
            for _ in range(128):
                p_full[g].arrive()
            nt += 1
        if T > 0:
            yield from wait(acc_full, 0)

    agents = [producer(), issuer(), compute(0), compute(1)]
    alive = list(range(len(agents)))
    stalls = 0
    while alive or pipe:
        choices = [("agent", a) for a in alive] + ([("pipe", 0)] if pipe else [])
        kind, who = rng.choice(choices)
        if kind == "pipe":
            k, val = pipe.pop(0)
            if k == "mma":
                pending[val] -= 1
            elif k == "write_tm":
                if pending.get(("tm", val, tm_uses[val] - 1), 0):
                    raise ProtocolError(f"S^T of group {val} written under a pending product")
            else:
                val.arrive()
            stalls = 0
            continue
        try:
            next(agents[who])
            stalls += 1
        except StopIteration:
            alive.remove(who)
            stalls = 0
        if stalls > 20000:
            raise ProtocolError("deadlock: no agent can make progress")


@pytest.mark.parametrize("NR", [2, 4])
@pytest.mark.parametrize("T", [1, 2, 3, 4, 7, 12])
def test_dkv_pass_protocol_random_schedules(T, NR):
    for seed in range(200):
        simulate_dkv(seed, T, NR=NR)


def test_dkv_model_detects_an_early_next_product():
    """Issuing a group's next S^T before its softmax has read the current one is
    caught (as an overwrite, a parity-ambiguous wait or a deadlock)."""
    caught = 0
    for seed in range(100):
        try:
            simulate_dkv(seed, 6, early_next=True)
        except AssertionError:
            caught += 1
    assert caught > 0


def simulate_dq(seed, Ts, early_dp=False, early_s=False, per_parity=True, NK=3, NV=2, stat_early=False):
    """The query-stationary dQ pass (csrc/bwd_tc.cu), persistent: one CTA walks units
    of Ts[u] key tiles each (a unit without key tiles only writes zeros).  Q and dO of
    a unit are loaded once the last unit's last S and dP are done (stat_empty); K
    through an NK-stage ring and V through an NV-stage ring (V released after dP, K
    after dQ), with CTA-wide tile indices; S of tile j in TMEM buffer j & 1, dP in one
    buffer.  The issuer computes S(j+1) while the compute warps work on tile j, dP(j+1)
    once they hold dP(j) in registers (dp_read), and S(j+2) into the buffer dQ(j) has
    just read; a unit's first S and dP follow the last unit's products at once (its
    first dP after the last unit's last dP was read), and its first dQ product, which
    overwrites the accumulator, after the compute warps' dS of its first tile, which
    they write after their epilogue has read the accumulator.  MMAs complete in issue
    order.  Checked: the compute warps read S(j) and dP(j) of their own tile, dS(j) is
    what dQ(j) reads, the epilogue reads its own unit's accumulator, no ring slot or
    Q/dO buffer is refilled under a pending reader, no deadlock, no parity-ambiguous
    wait.  per_parity=False models a single dS barrier, which the compute warps can
    drive two phases past the issuer's wait; stat_early releases Q/dO one product too
    early."""
    if isinstance(Ts, int):
        Ts = [Ts]
    rng = random.Random(seed)
    a_full = Barrier("a_full", 1)
    stat_empty = Barrier("stat_empty", 1)
    N = {"K": NK, "V": NV}
    full = {x: [Barrier(f"{x}_full{s}", 1) for s in range(N[x])] for x in "KV"}
    empty = {x: [Barrier(f"{x}_empty{s}", 1) for s in range(N[x])] for x in "KV"}
    s_full = Barrier("s_full", 1)
    dp_read = Barrier("dp_read", 128)
    ds_full = [Barrier(f"ds_full{x}", 128) for x in range(2)]   # one per key-tile parity
    acc_full = Barrier("acc_full", 1)
    pipe = []
    pending = {}
    loads = {"K": [0] * NK, "V": [0] * NV}
    stat_loads = [0]
    sbuf = [None, None]                     # what each S buffer holds: ("S", j) or ("dS", j)
    dpbuf = [None]                          # the tile whose dP the dP buffer holds
    acc = [None]                            # the unit whose dQ products the accumulator holds

    def mma_read(key):
        pending[key] = pending.get(key, 0) + 1
        pipe.append(("read", key))

    def ring_read(x, j):
        mma_read((x, j % N[x], loads[x][j % N[x]] - 1))

    def producer():
        ka = jg = 0
        for T in Ts:
            if T == 0:
                continue
            if ka > 0:
                yield from wait(stat_empty, ka - 1)
            if pending.get(("stat", stat_loads[0] - 1), 0):
                raise ProtocolError("Q/dO replaced while an S or dP product still reads them")
            stat_loads[0] += 1
            yield
            a_full.arrive()
            for j in range(T):
                jj = jg + j
                for x in "KV":
                    st = jj % N[x]
                    if jj >= N[x]:
                        yield from wait(empty[x][st], jj // N[x] - 1)
                    if pending.get((x, st, loads[x][st] - 1), 0):
                        raise ProtocolError(f"{x} slot {st} refilled under a pending reader")
                    loads[x][st] += 1
                    yield
                    full[x][st].arrive()
            ka += 1
            jg += T

    def issuer():
        def issue_s(j):
            yield from wait(full["K"][j % NK], j // NK)
            ring_read("K", j)
            mma_read(("stat", stat_loads[0] - 1))
            pipe.append(("write_s", j))

        def issue_dp(j):
            yield from wait(full["V"][j % NV], j // NV)
            ring_read("V", j)
            mma_read(("stat", stat_loads[0] - 1))
            pipe.append(("write_dp", j))
            pipe.append(("commit", empty["V"][j % NV]))

        ka = jg = 0
        for u, T in enumerate(Ts):
            if T == 0:
                continue
            yield from wait(a_full, ka)
            yield from issue_s(jg)
            if jg > 0:
                yield from wait(dp_read, jg - 1)
            if stat_early and T == 1:
                pipe.append(("commit", stat_empty))
            yield from issue_dp(jg)
            pipe.append(("commit", s_full))
            if T == 1 and not stat_early:
                pipe.append(("commit", stat_empty))
            if T > 1:
                yield from issue_s(jg + 1)
            for j in range(T):
                jj = jg + j
                if j + 1 < T:
                    if not early_dp:
                        yield from wait(dp_read, jj)
                    if stat_early and j + 2 == T:
                        pipe.append(("commit", stat_empty))
                    yield from issue_dp(jj + 1)
                    pipe.append(("commit", s_full))
                    if j + 2 == T and not stat_early:
                        pipe.append(("commit", stat_empty))
                yield from wait(ds_full[jj & 1] if per_parity else ds_full[0], (jj >> 1) if per_parity else jj)
                if early_s and j + 2 < T:              # planted: S(j+2) before dQ(j) read dS(j)
                    yield from issue_s(jj + 2)
                ring_read("K", jj)
                pipe.append(("read_ds", jj))
                pipe.append(("dq", u))
                pipe.append(("commit", empty["K"][jj % NK]))
                if j == T - 1:
                    pipe.append(("commit", acc_full))
                if j + 2 < T and not early_s:
                    yield from issue_s(jj + 2)
            ka += 1
            jg += T

    def compute():
        ka = jg = 0
        for u, T in enumerate(Ts):
            for j in range(T):
                jj = jg + j
                yield from wait(s_full, jj)
                if dpbuf[0] != jj:
                    raise ProtocolError(f"compute of tile {jj} read dP of tile {dpbuf[0]}")
                yield
                for _ in range(128):
                    dp_read.arrive()
                if sbuf[jj & 1] != ("S", jj):
                    raise ProtocolError(f"compute of tile {jj} read {sbuf[jj & 1]} from S buffer {jj & 1}")
                yield
                sbuf[jj & 1] = ("dS", jj)
                for _ in range(128):
                    (ds_full[jj & 1] if per_parity else ds_full[0]).arrive()
            if T > 0:
                yield from wait(acc_full, ka)
                if acc[0] != u:
                    raise ProtocolError(f"epilogue of unit {u} read the accumulator of unit {acc[0]}")
                yield
                ka += 1
            jg += T

    agents = [producer(), issuer(), compute()]
    alive = list(range(len(agents)))
    stalls = 0
    while alive or pipe:
        choices = [("agent", a) for a in alive] + ([("pipe", 0)] if pipe else [])
        kind, who = rng.choice(choices)
        if kind == "pipe":
            k, val = pipe.pop(0)
            if k == "read":
                pending[val] -= 1
            elif k == "write_s":
                sbuf[val & 1] = ("S", val)
            elif k == "write_dp":
                dpbuf[0] = val
            elif k == "read_ds":
                if sbuf[val & 1] != ("dS", val):
                    raise ProtocolError(f"dQ product of tile {val} read {sbuf[val & 1]}")
            elif k == "dq":
                acc[0] = val
            else:
                val.arrive()
            stalls = 0
            continue
        try:
            next(agents[who])
            stalls += 1
        except StopIteration:
            alive.remove(who)
            stalls = 0
        if stalls > 20000:
            raise ProtocolError("deadlock: no agent can make progress")


@pytest.mark.parametrize("seed0", [0, 1000])
def test_dq_persistent_units_random_schedules(seed0):
    """Several units per CTA, some without key tiles, with random tile counts."""
    for seed in range(seed0, seed0 + 150):
        r = random.Random(seed)
        Ts = [r.choice([0, 1, 2, 3, 5]) for _ in range(r.randint(1, 5))]
        simulate_dq(seed, Ts)


def test_dq_model_detects_an_early_stat_release():
    """Releasing Q/dO before the unit's last dP product is issued lets the next
    unit's load replace them under that product on some schedule."""
    caught = 0
    for seed in range(300):
        try:
            simulate_dq(seed, [2, 3, 1, 2], stat_early=True)
        except AssertionError:
            caught += 1
    assert caught > 0


@pytest.mark.parametrize("rings", [(2, 2), (3, 2)], ids=["kv2", "k3_v2"])
@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 9])
def test_dq_pass_protocol_random_schedules(T, rings):
    for seed in range(200):
        simulate_dq(seed, T, NK=rings[0], NV=rings[1])


def test_dq_model_detects_a_single_ds_barrier():
    """One dS barrier for every key tile lets the compute warps finish tile j+1 before
    the issuer waits for tile j: a parity wait two phases behind."""
    caught = 0
    for seed in range(200):
        try:
            simulate_dq(seed, 5, per_parity=False)
        except AssertionError:
            caught += 1
    assert caught > 0


@pytest.mark.parametrize("mistake", ["early_dp", "early_s"])
def test_dq_model_detects_a_misordered_product(mistake):
    """dP(j+1) issued before the compute warps hold dP(j), or S(j+2) issued into the
    buffer before the dQ product has read dS(j) from it, is caught as a wrong buffer
    content, a parity-ambiguous wait or a deadlock."""
    caught = 0
    for seed in range(100):
        try:
            simulate_dq(seed, 5, **{mistake: True})
        except AssertionError:
            caught += 1
    assert caught > 0
