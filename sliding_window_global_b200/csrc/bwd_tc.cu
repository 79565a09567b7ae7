// bwd_tc.cu -- backward pass of banded sparse self-attention on sm_100a
// (tcgen05 tensor cores, bf16 operands, fp32 accumulation in TMEM).
//
// Gradients of o = softmax(scale q k^T + mask) v for an upstream gradient dout,
// through the chain rule of the softmax (the same key sets as the forward: the
// sliding window of "精读笔记：Big Bird" §3.2.1, dilated as on the Longformer page
// §二, causal as in SWAN-GPT §3.3(1); GQA heads share K/V):
//   p = exp(scale q.k - lse),  dp = dout . v,  Delta = rowsum(dout * o),
//   ds = p (dp - Delta),  dq = scale ds k,  dk = scale ds^T q,  dv = p^T dout.
//
// Three launches:
//   bwd_delta_kernel     Delta per query row (CUDA cores, one warp per row);
//   bwd_dq_kernel<D>     query-stationary: one CTA per 128-row query tile walks
//                        its band's key tiles: S = Q K^T and dP = dO V^T into
//                        TMEM, dS written back as bf16 over S, dQ += dS K;
//   bwd_dkv_kernel<D>    key-stationary: one CTA per 128-key tile walks the 64-row
//                        query tiles (of every query head of its GQA group) that
//                        reach it, two compute warpgroups taking alternate tiles:
//                        S^T = K Q^T and dP^T = V dO^T into the group's TMEM
//                        columns, P^T and dS^T as bf16 into shared memory, then
//                        dV += P^T dO and dK += dS^T Q.
// Neither needs atomics: every output row belongs to one CTA.  S and dP are
// computed by both passes (seven tile products instead of five), the price of
// keeping dQ out of the key-stationary pass's TMEM, which D = 128 fills.
//
// Warp roles of the dQ pass (192 threads): warps 0-3 compute (thread t owns TMEM
// lane t), warp 4 issues the TMA loads, warp 5 allocates TMEM and issues the MMAs;
// the dK/dV pass (320 threads) has two compute warpgroups, then the same two.
#include <type_traits>

#include "ptx.cuh"
#include "softmax_math.cuh"
#include "swa_kernels.h"
#include "bwd_kernels.h"

namespace swa {
namespace {

constexpr int kBThreads = 192;
constexpr uint32_t kBSub = 128 * 128;          // one 128-row x 128-byte swizzle sub-tile
constexpr float kBLog2e = 1.4426950408889634f;

template <int D>
struct BCfg {
  static constexpr uint32_t kTileBytes = 128u * D * 2u;
  // the stationary Q and dO tiles, then a ring of K tiles and a ring of V tiles.  V is
  // read only by dP and freed early; K, read by S and by dQ, gets one stage more, so
  // the load of K(j+2) starts while dQ(j) still runs
  static constexpr int NK = 3, NV = 2;
  static constexpr uint32_t kStat0 = 0;
  static constexpr uint32_t kStat1 = kTileBytes;
  static constexpr uint32_t kKRing = 2 * kTileBytes;
  static constexpr uint32_t kVRing = kKRing + NK * kTileBytes;
  static constexpr uint32_t kBarOff = kVRing + NV * kTileBytes;
  static constexpr uint32_t kSmemBytes = kBarOff + 16 * 8 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  // TMEM columns (dQ pass): S of even key tiles 0-127 and of odd ones 384-511 (dS written
  // over its first 64 columns), dP 128-255, dQ from 256.
  static constexpr uint32_t kS = 0, kDP = 128, kAcc0 = 256, kS1 = 384;
  __host__ __device__ static constexpr uint32_t s_buf(int j) { return (j & 1) ? kS1 : kS; }
};

// dynamic shared memory plus the kernel's static arrays (sGpos, TMEM slot, abort flag)
static_assert(BCfg<128>::kSmemBytes + kTile * 4 + 16 <= 227 * 1024, "shared memory of the dQ pass");

// TMA load of one 128 x D bf16 tile (two 64-column boxes when D = 128).
template <int D>
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int y,
                                          int z) {
  tma_load_3d(dst, map, bar, 0, y, z);
  if (D == 128) tma_load_3d(dst + kBSub, map, bar, 64, y, z);
}

// S = A B^T for two K-major 128 x D tiles (128-byte swizzle), into TMEM.
template <int D>
__device__ __forceinline__ void mma_abt(uint32_t dst, uint32_t a, uint32_t b) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);
  const uint32_t al = sdesc_lo(a, 16), bl = sdesc_lo(b, 16);   // descriptor low words
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = ((kk >> 2) * kBSub + (kk & 3) * 32) >> 4;
    umma_ss_lo(dst, al + off, bl + off, idesc, kk > 0 ? 1u : 0u);
  }
}

// C (+)= P X: P a 128 x 128 bf16 matrix in TMEM (packed two per column), X a
// 128 x D tile in shared memory read as an MN-major B operand.
template <int D>
__device__ __forceinline__ void mma_px(uint32_t dst, uint32_t p_tmem, uint32_t x, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, true);
  const uint32_t xl = sdesc_lo(x, kBSub);                      // descriptor low word
  const uint32_t first = accumulate ? 1u : 0u;
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) umma_ts_lo(dst, p_tmem + kk * 8, xl + ((kk * 2048) >> 4), idesc, kk > 0 ? 1u : first);
}

struct BUnit {
  bool valid;
  int b, h, hk, cls, c, d, r, nc, Vc;
  int u0, rows, nvalid;   // the stationary tile (class coordinates)
};

// unit -> (b, head, class, tile); heads fastest.  `heads` = Hq (dQ) or Hkv (dKV).
__device__ __forceinline__ void decode_bunit(const BwdParams& p, int uid, bool kv_pass, BUnit& u) {
  const int heads = kv_pass ? p.Hkv : p.Hq;
  const int bh = uid % (p.B * heads);
  int t = uid / (p.B * heads);
  u.b = bh / heads;
  const int hh = bh % heads;
  u.h = kv_pass ? hh * p.G : hh;          // a query head (the group's first for dKV)
  u.hk = kv_pass ? hh : hh / p.G;
  u.valid = t < (kv_pass ? p.ktiles[hh] : p.qtiles[hh]);
  const int base = p.class_base[u.h];
  u.d = p.cls[base].d;
  u.r = p.window[u.h];
  const int nres = p.cls[base].nres;
  int c = 0;
  for (; c < nres - 1; ++c) {
    const int tc = (p.cls[base + c].n_c + kTile - 1) / kTile;
    if (t < tc) break;
    t -= tc;
  }
  u.c = c;
  u.cls = base + c;
  u.nc = p.cls[u.cls].n_c;
  int V = p.valid_len ? p.valid_len[u.b] : p.n;
  V = min(V, p.n);
  u.Vc = V > c ? (V - c + u.d - 1) / u.d : 0;
  u.u0 = t * kTile;
  u.rows = u.valid ? max(0, min(kTile, u.nc - u.u0)) : 0;
  u.nvalid = max(0, min(u.rows, u.Vc - u.u0));
}

__device__ __forceinline__ size_t pos_row(const BwdParams& p, const BUnit& u, int head, int heads, int uc) {
  return ((size_t)u.b * heads + head) * p.n + (size_t)(u.c + u.d * uc);
}

// ------------------------------------------------------------------ Delta
// One warp per two rows: every lane loads its D/32 elements of both rows of out and
// dout with one vector load each before any arithmetic, so four loads per lane are in
// flight (the pass is bound by HBM bandwidth).
template <int D>
__global__ void bwd_delta_kernel(const __grid_constant__ BwdParams p) {
  using V = typename std::conditional<D == 128, uint2, uint32_t>::type;   // D / 32 bf16
  const size_t warp = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const size_t rows = (size_t)p.B * p.Hq * p.n;
  const size_t r0 = 2 * warp;
  if (r0 >= rows) return;
  const bool two = r0 + 1 < rows;
  const V* o = reinterpret_cast<const V*>(static_cast<const __nv_bfloat16*>(p.out) + r0 * D) + lane;
  const V* g = reinterpret_cast<const V*>(static_cast<const __nv_bfloat16*>(p.dout) + r0 * D) + lane;
  constexpr int kPerRow = D / 64;                  // bf16 pairs per lane and row
  V oa = __ldg(o), ga = __ldg(g), ob = oa, gb = ga;
  if (two) {
    ob = __ldg(o + 32);
    gb = __ldg(g + 32);
  }
  float acc[2] = {0.f, 0.f};
  const V ov[2] = {oa, ob}, gv[2] = {ga, gb};
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const uint32_t* ow = reinterpret_cast<const uint32_t*>(&ov[r]);
    const uint32_t* gw = reinterpret_cast<const uint32_t*>(&gv[r]);
#pragma unroll
    for (int e = 0; e < kPerRow; ++e) {
      const float2 of = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ow[e]));
      const float2 gf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[e]));
      acc[r] = fmaf(of.x, gf.x, acc[r]);
      acc[r] = fmaf(of.y, gf.y, acc[r]);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], off);
    acc[1] += __shfl_xor_sync(0xffffffffu, acc[1], off);
  }
  if (lane == 0) {
    p.delta[r0] = acc[0];
    if (two) p.delta[r0 + 1] = acc[1];
  }
}

// ------------------------------------------------------------------ shared facts
// Position sets of the forward, written out per (query position, key position):
// the window W(i) of a head (radius r, dilation d, causal or not).
__device__ __forceinline__ bool in_window(int qpos, int kpos, int rd, int d, int causal) {
  const int diff = qpos - kpos;
  const bool span = causal ? (diff >= 0 && diff <= rd) : (diff >= -rd && diff <= rd);
  return span && (d == 1 || diff % d == 0);
}

// Is position `pos` one of batch b's global tokens?  (binary search: sorted list)
__device__ __forceinline__ bool is_global_pos(const BwdParams& p, int b, int pos) {
  if (p.g == 0) return false;
  const int32_t* gl = p.global_idx + (size_t)b * p.g;
  int lo = 0, hi = p.g;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    const int v = __ldg(gl + mid);
    if (v == pos) return true;
    if (v < pos) lo = mid + 1;
    else hi = mid;
  }
  return false;
}

__device__ __forceinline__ int batch_valid_len(const BwdParams& p, int b) {
  return min(p.valid_len ? __ldg(p.valid_len + b) : p.n, p.n);
}

// ------------------------------------------------------------------ dQ
// Query-stationary: a 128-row query tile (Q and dO resident) walks a list of key
// tiles through a two-stage ring.  X: after the band's tiles come the global-column
// tiles (gathered K/V of the global tokens), the side tiles and the random tiles of
// the row block, with the masks and biases of the forward; global query rows take
// only their window and side keys here.  GROWS: the stationary tile is 128 gathered
// global query rows, the key tiles are every tile of the sequence, and the mask keeps
// the keys outside each row's window; the result is added to dq.
// Units of the dQ pass: band, a 128-row query tile of one head's class (heads fastest);
// GROWS, a tile of 128 global slots of one head.  The kernel is persistent: CTA c takes
// units c, c + grid, ...
template <bool GROWS>
__device__ __forceinline__ int dq_units(const BwdParams& p) {
  return GROWS ? p.B * p.Hq * (p.gpad / kTile) : p.max_qtiles * p.B * p.Hq;
}

// Unit uid of the dQ pass and its key tiles: band tiles from klo_t (class
// coordinates), then (X) global-column, side and random tiles.  false: the unit has
// no rows (every role skips it).
template <bool X, bool GROWS>
__device__ __forceinline__ bool dq_unit(const BwdParams& p, int uid, BUnit& u, int& klo_t, int& T, int& nband,
                                        int& ngc, int& nside, int& nrand) {
  klo_t = T = nband = ngc = nside = nrand = 0;
  if (!GROWS) {
    decode_bunit(p, uid, false, u);
    if (!u.valid) return false;
    // band key range of the tile: [klo_t, khi_t) in class coordinates
    const int last = u.u0 + u.nvalid - 1;
    klo_t = max(0, u.u0 - u.r);
    const int khi_t = u.nvalid > 0 ? (p.causal ? min(u.Vc, last + 1) : min(u.Vc, last + u.r + 1)) : klo_t;
    nband = khi_t > klo_t ? (khi_t - klo_t + kTile - 1) / kTile : 0;
    if (X && u.nvalid > 0) {
      ngc = p.g > 0 ? (p.g + kTile - 1) / kTile : 0;
      nside = p.S > 0 ? (p.S + kTile - 1) / kTile : 0;
      nrand = p.rand_blocks ? p.num_rand : 0;
    }
    T = nband + ngc + nside + nrand;
  } else {
    // global rows: unit = (batch, query head, tile of 128 global slots)
    const int gtiles = p.gpad / kTile;
    const int bh = uid / gtiles, gt = uid % gtiles;
    u.valid = true;
    u.b = bh / p.Hq;
    u.h = bh % p.Hq;
    u.hk = u.h / p.G;
    u.cls = p.dense_class;
    u.c = 0;
    u.d = p.cls[p.class_base[u.h]].d;             // the head's own dilation, for its window
    u.r = p.window[u.h];
    u.nc = p.n;
    u.Vc = batch_valid_len(p, u.b);
    u.u0 = gt * kTile;
    u.rows = min(kTile, p.gpad - u.u0);
    u.nvalid = max(0, min(u.rows, p.g - u.u0));
    if (u.nvalid == 0) return false;
    T = (u.Vc + kTile - 1) / kTile;
    nband = T;
  }
  return true;
}

template <int D, bool X, bool GROWS>
__global__ void __launch_bounds__(kBThreads, 1) bwd_dq_kernel(const __grid_constant__ BwdParams p) {
  using C = BCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  constexpr int NK = C::NK, NV = C::NV;
  uint64_t* a_full = bars;          // Q and dO loaded
  uint64_t* s_full = bars + 1;      // S and dP in TMEM
  uint64_t* acc_full = bars + 2;    // dQ complete
  uint64_t* dp_read = bars + 3;     // dP read into registers (128 arrivals): the next dP may be written
  uint64_t* ds_full = bars + 4;     // [2] dS of even / odd key tiles written (128 arrivals): with
                                    // S and dP of tile j+1 issued before the wait for dS(j), the
                                    // compute warps may finish tile j+1 first; one barrier per parity
                                    // keeps every wait at most one phase behind
  uint64_t* k_full = bars + 6;      // [NK] K tile of a stage loaded
  uint64_t* k_empty = k_full + NK;  // [NK] its dQ product completed
  uint64_t* v_full = k_empty + NK;  // [NV] V tile of a stage loaded
  uint64_t* v_empty = v_full + NV;  // [NV] its dP product completed
  uint64_t* stat_empty = v_empty + NV;  // the unit's last S and dP done: Q, dO may be replaced
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int sGpos[kTile];      // key positions of the current global-column tile
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int nunits = dq_units<GROWS>(p);

  if (tid == 0) {
    mbar_init(a_full, 1);
    for (int s = 0; s < NK; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(&ds_full[0], 128);
    mbar_init(&ds_full[1], 128);
    mbar_init(acc_full, 1);
    mbar_init(dp_read, 128);
    mbar_init(stat_empty, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(&tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int* abort_v = &abort_flag;
  grid_dependency_wait();           // Delta (and the gathered rows) of the kernels before
  const int nqb = (p.n + kTile - 1) / kTile;
  // Every role walks the same units in the same order and keeps the same counters:
  // ka, units with key tiles so far (phases of a_full, stat_empty, acc_full), and jg,
  // key tiles so far (ring stages, S buffers and the per-tile barriers' phases).
  BUnit u;
  int klo_t, T, nband, ngc, nside, nrand;

  if (warp == 4) {
    if (lane == 0) {
      bool ok = true;
      int ka = 0, jg = 0;
      for (int uid = blockIdx.x; ok && uid < nunits; uid += gridDim.x) {
      if (!dq_unit<X, GROWS>(p, uid, u, klo_t, T, nband, ngc, nside, nrand) || T == 0) continue;
      const int qz = u.b * p.Hq + u.h;
      const int kz = u.b * p.Hkv + u.hk;
      const int qb = u.u0 / kTile;                 // query block of the tile (random blocks: d = 1)
      // Q and dO of this unit replace the last unit's once its last S and dP are done
      if (ka > 0 && !mbar_wait_bounded(stat_empty, (ka - 1) & 1, abort_v, kWaitLimitNs)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(a_full, 2 * C::kTileBytes);
      load_tile<D>(smem + C::kStat0, GROWS ? &p.mgq : &p.mq[u.cls], a_full, u.u0, qz);
      load_tile<D>(smem + C::kStat1, GROWS ? &p.mgdo : &p.mdo[u.cls], a_full, u.u0, qz);
      for (int j = 0; j < T; ++j) {
        const int jj = jg + j;                     // ring position
        const int sk = jj % NK, sv = jj % NV;
        if (jj >= NK && !mbar_wait_bounded(&k_empty[sk], ((jj / NK) - 1) & 1, abort_v, kWaitLimitNs)) {
          ok = false;
          break;
        }
        const CUtensorMap *mk = &p.mk[u.cls], *mv = &p.mv[u.cls];
        int y = GROWS ? j * kTile : klo_t + j * kTile;
        if (X && j >= nband) {
          if (j < nband + ngc) {
            mk = &p.mgk; mv = &p.mgv; y = (j - nband) * kTile;
          } else if (j < nband + ngc + nside) {
            mk = &p.msk; mv = &p.msv; y = (j - nband - ngc) * kTile;
          } else {
            const int t = j - nband - ngc - nside;
            y = __ldg(p.rand_blocks + (((size_t)u.b * p.Hq + u.h) * nqb + qb) * p.num_rand + t) * kTile;
          }
        }
        mbar_arrive_expect_tx(&k_full[sk], C::kTileBytes);
        load_tile<D>(smem + C::kKRing + sk * C::kTileBytes, mk, &k_full[sk], y, kz);
        if (jj >= NV && !mbar_wait_bounded(&v_empty[sv], ((jj / NV) - 1) & 1, abort_v, kWaitLimitNs)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&v_full[sv], C::kTileBytes);
        load_tile<D>(smem + C::kVRing + sv * C::kTileBytes, mv, &v_full[sv], y, kz);
      }
      ++ka;
      jg += T;
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      // Pipelined: S of tile j+1 is computed into the other S buffer while the compute
      // warps work on tile j, and dP of tile j+1 as soon as they have read dP of tile j,
      // so the next tile's products are ready when the compute warps are.  In issue
      // order (MMAs complete in order): a new S goes into the buffer whose dS the
      // previous dQ product read; a new dP after dp_read.  Indices are CTA-wide (jg +
      // j), so a unit's first S and dP follow the last unit's products at once and
      // overlap its last dS and its epilogue; the first dQ product of a unit, which
      // overwrites the accumulator, waits for the compute warps' dS of its first tile,
      // which they write after their epilogue has read the accumulator.
      const uint32_t qa = smem_u32(smem + C::kStat0), da = smem_u32(smem + C::kStat1);
      auto kstage = [&](int j) { return smem_u32(smem + C::kKRing + (j % NK) * C::kTileBytes); };
      auto issue_s = [&](int j) -> bool {           // S(j) = Q K(j)^T
        if (!mbar_wait_bounded(&k_full[j % NK], (j / NK) & 1, abort_v, kWaitLimitNs)) return false;
        tc_fence_after();
        mma_abt<D>(tmem + C::s_buf(j), qa, kstage(j));
        return true;
      };
      auto issue_dp = [&](int j) -> bool {          // dP(j) = dO V(j)^T; V(j) is then free
        if (!mbar_wait_bounded(&v_full[j % NV], (j / NV) & 1, abort_v, kWaitLimitNs)) return false;
        tc_fence_after();
        mma_abt<D>(tmem + C::kDP, da, smem_u32(smem + C::kVRing + (j % NV) * C::kTileBytes));
        umma_commit(&v_empty[j % NV]);
        return true;
      };
      bool ok = true;
      int ka = 0, jg = 0;
      for (int uid = blockIdx.x; ok && uid < nunits; uid += gridDim.x) {
        if (!dq_unit<X, GROWS>(p, uid, u, klo_t, T, nband, ngc, nside, nrand) || T == 0) continue;
        ok = mbar_wait_bounded(a_full, ka & 1, abort_v, kWaitLimitNs);
        if (ok) ok = issue_s(jg);
        // dP of the first tile replaces the last unit's last dP once it is in registers
        if (ok && jg > 0) ok = mbar_wait_bounded(dp_read, (jg - 1) & 1, abort_v, kWaitLimitNs);
        if (ok) ok = issue_dp(jg);
        if (ok) {
          umma_commit(s_full);
          if (T == 1) umma_commit(stat_empty);       // the unit's last S and dP
        }
        if (ok && T > 1) ok = issue_s(jg + 1);
        for (int j = 0; ok && j < T; ++j) {
          const int jj = jg + j;
          if (j + 1 < T) {
            // dP(j+1) once the compute warps hold dP(j) in registers
            if (!mbar_wait_bounded(dp_read, jj & 1, abort_v, kWaitLimitNs)) { ok = false; break; }
            if (!issue_dp(jj + 1)) { ok = false; break; }
            umma_commit(s_full);                     // S(j+1) and dP(j+1)
            if (j + 2 == T) umma_commit(stat_empty); // the unit's last S and dP
          }
          // dQ += dS(j) K(j), then the stage of tile j may be refilled
          if (!mbar_wait_bounded(&ds_full[jj & 1], (jj >> 1) & 1, abort_v, kWaitLimitNs)) { ok = false; break; }
          tc_fence_after();
          mma_px<D>(tmem + C::kAcc0, tmem + C::s_buf(jj), kstage(jj), j > 0);
          umma_commit(&k_empty[jj % NK]);
          if (j == T - 1) umma_commit(acc_full);
          if (j + 2 < T) ok = issue_s(jj + 2);         // into the buffer dQ(j) just read
        }
        ++ka;
        jg += T;
      }
    }
  } else {
    // ------------------------------------------------------------ compute
    const int row = tid;                       // TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    bool ok = true;
    int ka = 0, jg = 0;
    for (int uid = blockIdx.x; ok && uid < nunits; uid += gridDim.x) {
    if (!dq_unit<X, GROWS>(p, uid, u, klo_t, T, nband, ngc, nside, nrand)) continue;
    const int qb = u.u0 / kTile;               // query block of the tile (random blocks: d = 1)
    const bool row_valid = row < u.nvalid;
    const int uq = u.u0 + row;
    const int rd = u.r * u.d;
    // the row's position; band rows: class coordinates -> position; global rows: gathered
    int qpos = u.c + u.d * uq;
    if (GROWS) qpos = row_valid ? __ldg(p.global_idx + (size_t)u.b * p.g + uq) : 0;
    const int klo = uq - u.r;
    const int khi = row_valid ? min(p.causal ? uq : uq + u.r, u.Vc - 1) + 1 : klo;
    size_t prow = 0;
    float lse2 = 0.f, delta = 0.f;
    if (row < u.rows && (!GROWS || row_valid)) {
      prow = GROWS ? ((size_t)u.b * p.Hq + u.h) * p.n + qpos : pos_row(p, u, u.h, p.Hq, uq);
      if (row_valid) {
        lse2 = p.lse[prow] * kBLog2e;
        delta = p.delta[prow];
      }
    }
    // terms beyond the band (X): the row's facts
    bool row_global = false;
    const float* lrow = nullptr;               // local-bias table of the head at offset 0
    const float* srow = nullptr;               // side-bias row of the row's query block
    int rbl[kMaxRand];
#pragma unroll
    for (int t = 0; t < kMaxRand; ++t) rbl[t] = -1;
    if (X) {
      row_global = row_valid && is_global_pos(p, u.b, qpos);
      if (p.local_bias && !row_global)
        lrow = p.local_bias + (size_t)u.h * (2 * p.local_radius + 1) + p.local_radius;
      if (p.bias && p.S > 0)
        srow = p.bias + (size_t)u.h * (p.S + p.nblk - 1) + (p.nblk - 1 - qpos / p.side_block);
#pragma unroll
      for (int t = 0; t < kMaxRand; ++t)
        if (t < nrand) rbl[t] = __ldg(p.rand_blocks + (((size_t)u.b * p.Hq + u.h) * nqb + qb) * p.num_rand + t);
    }
    const float sl2 = p.scale_log2;
    for (int j = 0; j < T; ++j) {
      const int jj = jg + j;                   // CTA-wide tile index: barrier phases, S buffer
      // tile kind: 0 band (or every key, GROWS), 1 global columns, 2 side, 3 random
      int kind = 0, base = 0, t_rand = 0;
      if (X && j >= nband) {
        if (j < nband + ngc) { kind = 1; base = (j - nband) * kTile; }
        else if (j < nband + ngc + nside) { kind = 2; base = (j - nband - ngc) * kTile; }
        else { kind = 3; t_rand = j - nband - ngc - nside; }
      }
      if (X && kind == 1) {
        // stage the tile's global key positions: -1 for empty slots and for keys a
        // random block of this row block already counts (the forward's rule)
        int cv = base + row < p.g ? __ldg(p.global_idx + (size_t)u.b * p.g + base + row) : -1;
#pragma unroll
        for (int t = 0; t < kMaxRand; ++t)
          if (cv >= 0 && rbl[t] >= 0 && (cv >> 7) == rbl[t]) cv = -1;
        named_barrier_sync(1, 128);            // readers of the previous tile are done
        sGpos[row] = cv;
        named_barrier_sync(1, 128);
      }
      int kb = 0;
      bool dup = false;
      if (X && kind == 3) {
#pragma unroll
        for (int t = 0; t < kMaxRand; ++t)
          if (t == t_rand) kb = rbl[t];
#pragma unroll
        for (int t = 0; t < kMaxRand; ++t) dup = dup || (t < t_rand && rbl[t] == kb);
        dup = dup || kb < 0 || kb >= nqb;
      }
      if (!mbar_wait_bounded(s_full, jj & 1, abort_v, kWaitLimitNs)) { ok = false; break; }
      tc_fence_after();
      const int kv0 = GROWS ? j * kTile : (kind == 3 ? kb * kTile : klo_t + j * kTile);
      const int lo_t = klo - kv0, hi_t = khi - kv0;
      // dP of the tile into registers, then its TMEM columns go back to the MMA warp
      uint32_t dpr[kTile];
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) tmem_ld32(lane_base + C::kDP + ch * 32, *reinterpret_cast<uint32_t(*)[32]>(dpr + ch * 32));
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) tmem_wait_ld_dep(*reinterpret_cast<uint32_t(*)[32]>(dpr + ch * 32));
      tc_fence_before();
      mbar_arrive(dp_read);
      const uint32_t sb = lane_base + C::s_buf(jj);
      // Interior band tile: every key of the tile is in the window of every row of this
      // warp, so no element needs a mask, and pairs of columns take one packed f32x2
      // instruction per step.
      // (the condition is warp-uniform outside the vote: kind depends only on j)
      const bool interior = !GROWS && (!X || kind == 0) &&
                            __all_sync(0xffffffffu, (!X || !lrow) && lo_t <= 0 && hi_t >= kTile);
      const float nl2 = -lse2, nd = -delta;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t sr[32];
        tmem_ld32(sb + ch * 32, sr);
        tmem_wait_ld_dep(sr);
        const uint32_t* dr = dpr + ch * 32;
        uint32_t pk[16];
        if (interior) {
#pragma unroll
          for (int q = 0; q < 32; q += 2) {
            float a0, a1, t0, t1, d0, d1;
            ffma2(a0, a1, __uint_as_float(sr[q]), __uint_as_float(sr[q + 1]), sl2, sl2, nl2, nl2);
            a0 = ex2_approx(a0);
            a1 = ex2_approx(a1);
            fadd2(t0, t1, __uint_as_float(dr[q]), __uint_as_float(dr[q + 1]), nd, nd);
            ffma2(d0, d1, a0, a1, t0, t1, 0.f, 0.f);
            pk[q / 2] = pack_bf16x2(d0, d1);
          }
          tmem_st16(sb + ch * 16, pk);
          continue;
        }
        // the packed steps of the interior; keys the predicate rejects give p = 0
        auto masked_packed = [&](auto allow) {
#pragma unroll
          for (int q = 0; q < 32; q += 2) {
            const int e = ch * 32 + q;
            float a0, a1, t0, t1, d0, d1;
            ffma2(a0, a1, __uint_as_float(sr[q]), __uint_as_float(sr[q + 1]), sl2, sl2, nl2, nl2);
            a0 = allow(e) ? ex2_approx(a0) : 0.f;
            a1 = allow(e + 1) ? ex2_approx(a1) : 0.f;
            fadd2(t0, t1, __uint_as_float(dr[q]), __uint_as_float(dr[q + 1]), nd, nd);
            ffma2(d0, d1, a0, a1, t0, t1, 0.f, 0.f);
            pk[q / 2] = pack_bf16x2(d0, d1);
          }
        };
        // band boundary tile: keys outside the row's window [lo_t, hi_t), one unsigned
        // compare each
        auto band_packed = [&]() {
          const unsigned span = (unsigned)max(hi_t - lo_t, 0);
          masked_packed([&](int e) { return (unsigned)(e - lo_t) < span; });
        };
        // Without dilation and the causal cut, "outside the row's window" is one unsigned
        // compare: (unsigned)(qpos + rd - key) > 2 rd.
        const unsigned span2 = 2u * (unsigned)rd;
        // per-element path: every tile kind, with its masks and biases
        auto generic_path = [&]() {
#pragma unroll
          for (int q = 0; q < 32; q += 2) {
            float ds[2];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int e = ch * 32 + q + h2;
              bool allowed;
              float b2 = 0.f;                    // bias in log2 units
              if (GROWS) {
                const int key = kv0 + e;
                allowed = row_valid && key < u.Vc && !in_window(qpos, key, rd, u.d, p.causal);
              } else if (!X || kind == 0) {
                allowed = e >= lo_t && e < hi_t;
                if (X && lrow && allowed) b2 = __ldg(lrow + u.d * (kv0 + e - uq)) * kBLog2e;
              } else if (kind == 1) {
                const int cv = sGpos[e];
                allowed = row_valid && !row_global && cv >= 0 && !in_window(qpos, cv, rd, u.d, p.causal);
              } else if (kind == 2) {
                const int sg = base + e;
                allowed = row_valid && sg < p.S;
                if (srow && allowed) b2 = __ldg(srow + sg) * kBLog2e;
              } else {
                const int key = kv0 + e;
                allowed = row_valid && !row_global && !dup && key < u.Vc &&
                          !in_window(qpos, key, rd, 1, p.causal);
              }
              const float pr = allowed ? ex2_approx(__uint_as_float(sr[q + h2]) * sl2 + b2 - lse2) : 0.f;
              ds[h2] = pr * (__uint_as_float(dr[q + h2]) - delta);
            }
            pk[q / 2] = pack_bf16x2(ds[0], ds[1]);
          }
        };
        if constexpr (GROWS) {
          if (!p.causal && (u.d & (u.d - 1)) == 0) {
            // a global row over every key tile: valid keys outside its window, i.e. not
            // within rd of the row or (dilation a power of two) of another residue class
            const int vlim = row_valid ? u.Vc - kv0 : 0;
            const int br = qpos + rd - kv0;
            const unsigned dm = (unsigned)u.d - 1u;
            masked_packed([&](int e) {
              return e < vlim && ((unsigned)(br - e) > span2 || ((unsigned)(br - e) & dm) != 0u);
            });
          } else {
            generic_path();
          }
        } else if constexpr (!X) {
          band_packed();
        } else if (kind == 0 && !p.local_bias) {
          band_packed();
        } else if (kind == 0) {
          // band tile with the local bias: keys of the row's window [lo_t, hi_t), each
          // with the bias of its offset (none for a global row, lrow = null)
          const unsigned span = (unsigned)max(hi_t - lo_t, 0);
#pragma unroll
          for (int q = 0; q < 32; q += 2) {
            const int e = ch * 32 + q;
            const bool in0 = (unsigned)(e - lo_t) < span, in1 = (unsigned)(e + 1 - lo_t) < span;
            float b0 = 0.f, b1 = 0.f;
            if (lrow) {
              b0 = in0 ? __ldg(lrow + u.d * (kv0 + e - uq)) : 0.f;
              b1 = in1 ? __ldg(lrow + u.d * (kv0 + e + 1 - uq)) : 0.f;
            }
            float a0, a1, t0, t1, d0, d1;
            ffma2(a0, a1, b0, b1, kBLog2e, kBLog2e, nl2, nl2);
            ffma2(a0, a1, __uint_as_float(sr[q]), __uint_as_float(sr[q + 1]), sl2, sl2, a0, a1);
            a0 = in0 ? ex2_approx(a0) : 0.f;
            a1 = in1 ? ex2_approx(a1) : 0.f;
            fadd2(t0, t1, __uint_as_float(dr[q]), __uint_as_float(dr[q + 1]), nd, nd);
            ffma2(d0, d1, a0, a1, t0, t1, 0.f, 0.f);
            pk[q / 2] = pack_bf16x2(d0, d1);
          }
        } else if (kind == 2) {
          // side tile: p = 2^(s scale log2e + bias log2e - lse log2e) for side keys below
          // S (every valid row attends them), packed steps; the bias of each key is read
          // from the row's side-bias row
          const int lim = row_valid ? p.S - base : 0;
#pragma unroll
          for (int q = 0; q < 32; q += 2) {
            const int e = ch * 32 + q;
            float b0 = 0.f, b1 = 0.f;
            if (srow) {
              b0 = e < lim ? __ldg(srow + base + e) : 0.f;
              b1 = e + 1 < lim ? __ldg(srow + base + e + 1) : 0.f;
            }
            float a0, a1, t0, t1, d0, d1;
            ffma2(a0, a1, b0, b1, kBLog2e, kBLog2e, nl2, nl2);
            ffma2(a0, a1, __uint_as_float(sr[q]), __uint_as_float(sr[q + 1]), sl2, sl2, a0, a1);
            a0 = e < lim ? ex2_approx(a0) : 0.f;
            a1 = e + 1 < lim ? ex2_approx(a1) : 0.f;
            fadd2(t0, t1, __uint_as_float(dr[q]), __uint_as_float(dr[q + 1]), nd, nd);
            ffma2(d0, d1, a0, a1, t0, t1, 0.f, 0.f);
            pk[q / 2] = pack_bf16x2(d0, d1);
          }
        } else if (kind == 1 && !p.causal && (u.d & (u.d - 1)) == 0) {
          // global-column tile: staged keys (-1: none, or counted by a random block)
          // outside the row's window (not within rd, or of another residue class when
          // the dilation is a power of two), for rows that are not global themselves
          const bool row_ok = row_valid && !row_global;
          const int qr = qpos + rd;
          const unsigned dm = (unsigned)u.d - 1u;
          masked_packed([&](int e) {
            const int cv = sGpos[e];
            return row_ok && cv >= 0 && ((unsigned)(qr - cv) > span2 || ((unsigned)(qr - cv) & dm) != 0u);
          });
        } else if (kind == 3 && !p.causal) {
          // random tile (dilation 1): valid keys of a first occurrence of the block,
          // outside the row's window, for rows that are not global
          const int vlim = (row_valid && !row_global && !dup) ? u.Vc - kv0 : 0;
          const int br = qpos + rd - kv0;
          masked_packed([&](int e) { return e < vlim && (unsigned)(br - e) > span2; });
        } else {
          generic_path();
        }
        // dS as bf16 over S: chunk ch writes columns 16ch.. that earlier chunks read
        tmem_st16(sb + ch * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&ds_full[jj & 1]);
    }
    // epilogue: dQ = scale * (dS K), fp32; padded rows get zeros.  Global rows (GROWS)
    // add their part to what the band pass wrote.
    if (ok && T > 0) ok = mbar_wait_bounded(acc_full, ka & 1, abort_v, kWaitLimitNs);
    if (ok) {
      tc_fence_after();
      float* dst = p.dq + prow * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t rr[32];
        if (T > 0) {
          tmem_ld32(lane_base + C::kAcc0 + ch * 32, rr);
          tmem_wait_ld_dep(rr);
        }
        if (GROWS ? row_valid : row < u.rows) {
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (T > 0 && row_valid)
              v4 = make_float4(__uint_as_float(rr[q4 * 4]) * p.scale, __uint_as_float(rr[q4 * 4 + 1]) * p.scale,
                               __uint_as_float(rr[q4 * 4 + 2]) * p.scale, __uint_as_float(rr[q4 * 4 + 3]) * p.scale);
            float4* d4 = reinterpret_cast<float4*>(dst) + ch * 8 + q4;
            if (GROWS) {
              const float4 o = *d4;
              v4 = make_float4(o.x + v4.x, o.y + v4.y, o.z + v4.z, o.w + v4.w);
            }
            *d4 = v4;
          }
        }
      }
    }
    if (T > 0) ++ka;
    jg += T;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (abort_flag) {
    if (tid == 0) {
      atomicOr(p.err, kDevErrTimeout);
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < 2000000ull) {
      }
    }
    __syncthreads();
  }
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------------ dK, dV
// Key-stationary pass with 64-row query tiles and two compute warpgroups that take
// alternate query tiles, each with its own S^T / dP^T columns in TMEM (M = 128 keys,
// N = 64 queries), so one group's exponentials overlap the other group's products.
// P^T and dS^T are written as bf16 over the columns of S^T and dP^T and feed
// dV += P^T dO and dK += dS^T Q as TMEM operands (A = 128 keys x 64 queries).
constexpr int kQT = 64;                        // query rows per tile of this pass
constexpr int kMaxRandList = 2048;             // (query head in group, query block) pairs per key block
constexpr int kDkvThreads = 320;               // warps 0-3, 4-7 compute; 8 TMA; 9 MMA / TMEM

template <int D>
struct KCfg {
  static constexpr uint32_t kKVBytes = 128u * D * 2u;      // a 128 x D tile
  static constexpr uint32_t kQBytes = kQT * D * 2u;        // a 64 x D tile
  static constexpr uint32_t kQSub = kQT * 128u;            // 64-row x 128-byte sub-tile
  static constexpr uint32_t kK = 0, kV = kKVBytes;
  // Q / dO ring: a tile's load starts when the products of the tile NR earlier are
  // done, so with NR > 2 the next S^T of a group need not wait for its load
  static constexpr int NR = 4;
  static constexpr uint32_t kRing = 2 * kKVBytes;          // stage s: Q at kRing + 2 s Q, dO after
  static constexpr uint32_t kFlags = kRing + 2 * NR * kQBytes;  // random job: per-pair flags (set-up only)
  // [group][buffer][lse2 64 | delta 64 | position 64 | row fact 64] (floats, ints)
  static constexpr uint32_t kStg = kFlags + kMaxRandList * 4;
  static constexpr uint32_t kList = kStg + 2 * 2 * 256 * 4;  // random job: query blocks drawing the key block
  static constexpr uint32_t kBarOff = kList + kMaxRandList * 4;
  static constexpr uint32_t kSmemBytes = kBarOff + 16 * 8 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  // TMEM: group g S^T at 128 g (P^T over its first 32 columns), dP^T at 128 g + 64
  // (dS^T over its first 32); dV at 256, dK at 256 + D
  static constexpr uint32_t kAccV = 256, kAccK = 256 + D;
};
static_assert(KCfg<128>::kSmemBytes <= 227 * 1024, "shared memory of the dK/dV pass");

// Jobs of the key-stationary pass.
enum DkvJob {
  kJobBand = 0,        // band key tile of a class, its band query tiles (overwrites dk, dv)
  kJobBandX = 1,       // the same with the local bias, and the global query rows outside the
                       // key's window appended (gathered rows)
  kJobGlobalKeys = 2,  // gathered global keys: every query row of the sequence whose window,
                       // and whose row block's random blocks, miss the key (adds to dk, dv)
  kJobSide = 3,        // a side tile: every valid query row, with the side bias (dside_k, dside_v)
  kJobRandom = 4,      // a random key block: the rows of the query blocks that drew it (adds)
};

// Query tiles of one key-stationary unit.  A tile is 64 query rows of one query
// head of the unit's GQA group; `src` 0 reads the class view (band), 1 the gathered
// global rows, 2 the whole sequence (dense class).
struct QTile {
  int head, y, src;
};

template <int D, int JOB>
__global__ void __launch_bounds__(kDkvThreads, 1) bwd_dkv_kernel(const __grid_constant__ BwdParams p) {
  using C = KCfg<D>;
  constexpr bool kBandJob = JOB == kJobBand || JOB == kJobBandX;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  constexpr int NR = C::NR;
  uint64_t* a_full = bars;               // K and V loaded
  uint64_t* r_full = bars + 1;           // [NR] Q, dO of a ring stage loaded
  uint64_t* r_empty = r_full + NR;       // [NR] that stage's products are done
  uint64_t* s_full = r_empty + NR;       // [2] S^T, dP^T of group g in TMEM
  uint64_t* p_full = s_full + 2;         // [2] group g wrote P^T, dS^T (and read its TMEM), 128 arrivals
  uint64_t* acc_full = p_full + 2;       // dK, dV complete
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int sCount;
  int* sList = reinterpret_cast<int*>(smem + C::kList);   // random job: head-in-group * nqb + query block
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nqb = (p.n + kTile - 1) / kTile;

  BUnit u;
  int qlo = 0, NQ = 0, NG = 0, ND = 0, T = 0;
  int kpos0 = 0;                    // position of key row 0 (band: class coordinates handled below)
  if (kBandJob) {
    decode_bunit(p, blockIdx.x, true, u);
    if (!u.valid) return;
    const int lastk = u.u0 + u.nvalid - 1;
    qlo = p.causal ? u.u0 : max(0, u.u0 - u.r);
    const int qhi = u.nvalid > 0 ? min(u.Vc, lastk + u.r + 1) : qlo;
    NQ = qhi > qlo ? (qhi - qlo + kQT - 1) / kQT : 0;
    NG = (JOB == kJobBandX && p.g > 0 && u.nvalid > 0) ? (p.g + kQT - 1) / kQT : 0;
    T = (NQ + NG) * p.G;            // 64-row query tiles of every head of the group
  } else {
    // unit = (batch, KV head, key tile of the job's key set)
    int per = 0;
    if (JOB == kJobGlobalKeys) per = p.gpad / kTile;
    if (JOB == kJobSide) per = (p.S + kTile - 1) / kTile;
    if (JOB == kJobRandom) per = nqb;
    const int bk = blockIdx.x / per, kt = blockIdx.x % per;
    u.valid = true;
    u.b = bk / p.Hkv;
    u.hk = bk % p.Hkv;
    u.h = u.hk * p.G;
    u.cls = p.dense_class;
    u.c = 0;
    u.d = p.cls[p.class_base[u.h]].d;
    u.r = p.window[u.h];
    u.nc = p.n;
    u.Vc = batch_valid_len(p, u.b);
    u.u0 = kt * kTile;
    if (JOB == kJobGlobalKeys) {
      u.rows = min(kTile, p.gpad - u.u0);
      u.nvalid = max(0, min(u.rows, p.g - u.u0));
    } else if (JOB == kJobSide) {
      u.rows = min(kTile, p.S - u.u0);
      u.nvalid = u.rows;            // every side key; with no valid row T = 0 writes zeros
    } else {
      u.rows = min(kTile, p.n - u.u0);
      u.nvalid = max(0, min(u.rows, u.Vc - u.u0));
    }
    if (u.nvalid == 0) return;      // no key of this tile exists: nothing to add
    kpos0 = u.u0;
    ND = (u.Vc + kQT - 1) / kQT;
    if (JOB == kJobRandom) {
      // the (head, query block) pairs of the group whose random list names this key
      // block, each counted at its first occurrence; built in a fixed order
      const int pairs = p.G * nqb;
      int* flags = reinterpret_cast<int*>(smem + C::kFlags);
      if (pairs > kMaxRandList) {
        if (tid == 0) atomicOr(p.err, kDevErrCheck);   // more pairs than the list holds: reported
        return;
      }
      for (int i = tid; i < pairs; i += blockDim.x) {
        const int32_t* rl = p.rand_blocks + (((size_t)u.b * p.Hq + u.h + i / nqb) * nqb + i % nqb) * p.num_rand;
        int f = 0;
        for (int t = 0; t < p.num_rand; ++t) f |= (__ldg(rl + t) == kt);   // a repeat counts once
        flags[i] = f;
      }
      __syncthreads();
      if (warp == 0) {                                  // ordered compaction, 32 pairs a step
        int cnt = 0;
        for (int base = 0; base < pairs; base += 32) {
          const int i = base + lane;
          const bool f = i < pairs && flags[i];
          const unsigned m = __ballot_sync(0xffffffffu, f);
          if (f) sList[cnt + __popc(m & ((1u << lane) - 1u))] = i;
          cnt += __popc(m);
        }
        if (lane == 0) sCount = cnt;
      }
      __syncthreads();
      T = 2 * sCount;               // two 64-row halves per query block
    } else {
      T = ND * p.G;
    }
  }
  auto qtile = [&](int j) -> QTile {
    QTile t;
    if (kBandJob) {
      const int per = NQ + NG;
      t.head = u.h + j / per;
      const int jj = j % per;
      if (jj < NQ) { t.y = qlo + jj * kQT; t.src = 0; }
      else { t.y = (jj - NQ) * kQT; t.src = 1; }
    } else if (JOB == kJobRandom) {
      const int e = sList[j >> 1];
      t.head = u.h + e / nqb;
      t.y = (e % nqb) * kTile + (j & 1) * kQT;
      t.src = 2;
    } else {
      t.head = u.h + j / ND;
      t.y = (j % ND) * kQT;
      t.src = 2;
    }
    return t;
  };

  if (tid == 0) {
    mbar_init(a_full, 1);
    for (int s = 0; s < NR; ++s) {
      mbar_init(&r_full[s], 1);
      mbar_init(&r_empty[s], 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&s_full[g], 1);
      mbar_init(&p_full[g], 128);
    }
    mbar_init(acc_full, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(&tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int* abort_v = &abort_flag;
  grid_dependency_wait();           // the passes before: Delta, dq, and dk/dv that this job adds to
  const int kz = u.b * p.Hkv + u.hk;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && T > 0) {
      const CUtensorMap* km = JOB == kJobGlobalKeys ? &p.mgk : JOB == kJobSide ? &p.msk : &p.mk[u.cls];
      const CUtensorMap* vm = JOB == kJobGlobalKeys ? &p.mgv : JOB == kJobSide ? &p.msv : &p.mv[u.cls];
      mbar_arrive_expect_tx(a_full, 2 * C::kKVBytes);
      load_tile<D>(smem + C::kK, km, a_full, u.u0, kz);
      load_tile<D>(smem + C::kV, vm, a_full, u.u0, kz);
      for (int j = 0; j < T; ++j) {
        const int st = j % NR;
        if (j >= NR && !mbar_wait_bounded(&r_empty[st], ((j / NR) - 1) & 1, abort_v, kWaitLimitNs)) break;
        const QTile qt = qtile(j);
        const int qz = u.b * p.Hq + qt.head;
        const CUtensorMap* qm = qt.src == 0 ? &p.mq64[u.cls] : qt.src == 1 ? &p.mgq64 : &p.mq64[p.dense_class];
        const CUtensorMap* dm = qt.src == 0 ? &p.mdo64[u.cls] : qt.src == 1 ? &p.mgdo64 : &p.mdo64[p.dense_class];
        uint8_t* dst = smem + C::kRing + st * 2 * C::kQBytes;
        mbar_arrive_expect_tx(&r_full[st], 2 * C::kQBytes);
        tma_load_3d(dst, qm, &r_full[st], 0, qt.y, qz);
        if (D == 128) tma_load_3d(dst + C::kQSub, qm, &r_full[st], 64, qt.y, qz);
        tma_load_3d(dst + C::kQBytes, dm, &r_full[st], 0, qt.y, qz);
        if (D == 128) tma_load_3d(dst + C::kQBytes + C::kQSub, dm, &r_full[st], 64, qt.y, qz);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && T > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, kQT, false);    // S^T, dP^T: 128 x 64
      constexpr uint32_t idesc_a = idesc_bf16_f32(128, D, true);       // dV, dK: 128 x D, B MN-major
      const uint32_t ka = sdesc_lo(smem_u32(smem + C::kK), 16), va = sdesc_lo(smem_u32(smem + C::kV), 16);
      // S^T = K Q^T and dP^T = V dO^T of tile j into group (j & 1)'s columns
      auto issue_s = [&](int j) -> bool {
        const int st = j % NR, g = j & 1;
        if (!mbar_wait_bounded(&r_full[st], (j / NR) & 1, abort_v, kWaitLimitNs)) return false;
        tc_fence_after();
        const uint32_t qb = sdesc_lo(smem_u32(smem + C::kRing + st * 2 * C::kQBytes), 16);
        const uint32_t db = qb + (C::kQBytes >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t offa = ((kk >> 2) * kBSub + (kk & 3) * 32) >> 4;
          const uint32_t offb = ((kk >> 2) * C::kQSub + (kk & 3) * 32) >> 4;
          umma_ss_lo(tmem + 128 * g, ka + offa, qb + offb, idesc_s, kk > 0 ? 1u : 0u);
          umma_ss_lo(tmem + 128 * g + 64, va + offa, db + offb, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[g]);
        return true;
      };
      bool ok = mbar_wait_bounded(a_full, 0, abort_v, kWaitLimitNs);
      if (ok) ok = issue_s(0);
      if (ok && T > 1) ok = issue_s(1);
      for (int j = 0; ok && j < T; ++j) {
        const int g = j & 1, st = j % NR;
        if (!mbar_wait_bounded(&p_full[g], (j >> 1) & 1, abort_v, kWaitLimitNs)) { ok = false; break; }
        tc_fence_after();
        const uint32_t qb = sdesc_lo(smem_u32(smem + C::kRing + st * 2 * C::kQBytes), C::kQSub);
        const uint32_t db = qb + (C::kQBytes >> 4);
        const uint32_t first = j > 0 ? 1u : 0u;
        // dV += P^T dO, dK += dS^T Q (A: 128 x 64 bf16 from the group's TMEM columns,
        // 16 queries = 8 columns per product; B: 64 x D MN-major from shared memory)
#pragma unroll
        for (int kk = 0; kk < kQT / 16; ++kk) {
          umma_ts_lo(tmem + C::kAccV, tmem + 128 * g + kk * 8, db + ((kk * 2048) >> 4), idesc_a,
                     kk > 0 ? 1u : first);
          umma_ts_lo(tmem + C::kAccK, tmem + 128 * g + 64 + kk * 8, qb + ((kk * 2048) >> 4), idesc_a,
                     kk > 0 ? 1u : first);
        }
        umma_commit(&r_empty[st]);
        // The group has read its S^T, dP^T of tile j; the next ones overwrite the same
        // columns only after the products above have read P^T, dS^T (in-order pipe).
        if (j + 2 < T) ok = issue_s(j + 2);
      }
      if (ok) umma_commit(acc_full);
    }
  } else {
    // ------------------------------------------------------------ compute warpgroups
    const int g = warp >> 2;                  // takes query tiles j with j & 1 == g
    const int row = tid & 127;                // key row, TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const bool key_valid = row < u.nvalid;
    const int uk = u.u0 + row;
    const int rd = u.r * u.d;
    // the key's position (band jobs: class coordinates c + d * uk)
    int kpos = kBandJob ? u.c + u.d * uk : kpos0 + row;
    if (JOB == kJobGlobalKeys) kpos = key_valid ? __ldg(p.global_idx + (size_t)u.b * p.g + uk) : 0;
    const float sl2 = p.scale_log2;
    bool ok = true;
    int nt = 0;                               // tiles handled by this group
    for (int j = g; j < T; j += 2, ++nt) {
      // per query row of the tile: -lse2 (-inf excludes the row: padded, missing, or
      // outside the job's rows), -Delta, and the row's position or block facts
      const QTile qt = qtile(j);
      float* stg = reinterpret_cast<float*>(smem + C::kStg) + (g * 2 + (nt & 1)) * 256;
      int* stgi = reinterpret_cast<int*>(stg + 2 * kQT);   // [64] positions, [64] extra
      if (row < kQT) {
        const int uq = qt.y + row;
        float l2 = INFINITY, dl = 0.f;
        int qp = 0, ex = 0;
        bool take = false;
        if (qt.src == 0) {
          take = uq < u.Vc;
          qp = u.c + u.d * uq;
          // the local bias applies to the window keys of non-global rows
          if (JOB == kJobBandX) ex = (p.local_bias && take && !is_global_pos(p, u.b, qp)) ? 1 : 0;
        } else if (qt.src == 1) {
          take = uq < p.g;
          qp = take ? __ldg(p.global_idx + (size_t)u.b * p.g + uq) : 0;
        } else {
          take = uq < u.Vc;
          qp = uq;
          if (JOB == kJobGlobalKeys || JOB == kJobRandom) take = take && !is_global_pos(p, u.b, qp);
          // query block of the side bias (block 0 for rows that do not count, so that the
          // bias read of every column stays inside the table)
          if (JOB == kJobSide) ex = take ? qp / p.side_block : 0;
        }
        if (take) {
          const size_t pr = ((size_t)u.b * p.Hq + qt.head) * p.n + qp;
          l2 = p.lse[pr] * kBLog2e;
          dl = p.delta[pr];
        }
        stg[row] = -l2;                          // negated: the products below add them
        stg[kQT + row] = -dl;
        stgi[row] = qp;
        stgi[kQT + row] = ex;
      }
      // global-key job: the random blocks of the tile's query block (one block per tile)
      int trb[kMaxRand];
#pragma unroll
      for (int t = 0; t < kMaxRand; ++t) trb[t] = -1;
      if (JOB == kJobGlobalKeys && p.rand_blocks) {
        const int qbk = qt.y / kTile;
#pragma unroll
        for (int t = 0; t < kMaxRand; ++t)
          if (t < p.num_rand) trb[t] = __ldg(p.rand_blocks + (((size_t)u.b * p.Hq + qt.head) * nqb + qbk) * p.num_rand + t);
      }
      bool key_in_rand = false;
#pragma unroll
      for (int t = 0; t < kMaxRand; ++t) key_in_rand = key_in_rand || (trb[t] >= 0 && (kpos >> 7) == trb[t]);
      const float* lrow = (JOB == kJobBandX && p.local_bias)
                              ? p.local_bias + (size_t)qt.head * (2 * p.local_radius + 1) + p.local_radius
                              : nullptr;
      const float* sbias = (JOB == kJobSide && p.bias)
                               ? p.bias + (size_t)qt.head * (p.S + p.nblk - 1) + (p.nblk - 1) + uk
                               : nullptr;
      named_barrier_sync(1 + g, 128);
      if (!mbar_wait_bounded(&s_full[g], nt & 1, abort_v, kWaitLimitNs)) { ok = false; break; }
      tc_fence_after();
      const int d0 = qt.y - uk;                // query - key offset of column 0 (band, class coordinates)
      // Interior tile of the band job: every (key, query) pair of this warp's keys is in
      // the band, so no element needs a mask (query rows that do not count have
      // -lse2 = -inf and give p = 0 by themselves).  Pairs of columns then take one
      // packed f32x2 instruction per step.
      bool interior = false;
      if (JOB == kJobBand) {
        const bool in = key_valid && (p.causal ? (d0 >= 0 && d0 + kQT - 1 <= u.r)
                                               : (d0 >= -u.r && d0 + kQT - 1 <= u.r));
        interior = __all_sync(0xffffffffu, in);
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {   // 32 query columns at a time
        uint32_t sr[32], dr[32];
        uint32_t pk[16], dk[16];               // P^T, dS^T of the 32 columns as bf16 pairs
        tmem_ld32(lane_base + 128 * g + 32 * half, sr);
        tmem_ld32(lane_base + 128 * g + 64 + 32 * half, dr);
        tmem_wait_ld_dep(sr);
        tmem_wait_ld_dep(dr);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {       // 16-byte chunks of 8 queries
          const int c = half * 4 + c4;
          const float4 la = *reinterpret_cast<const float4*>(stg + c * 8);
          const float4 lb = *reinterpret_cast<const float4*>(stg + c * 8 + 4);
          const float4 da = *reinterpret_cast<const float4*>(stg + kQT + c * 8);
          const float4 db = *reinterpret_cast<const float4*>(stg + kQT + c * 8 + 4);
          const float lv[8] = {la.x, la.y, la.z, la.w, lb.x, lb.y, lb.z, lb.w};   // -lse2
          const float dv[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};   // -Delta
          float pr[8], ds[8];
          if (interior) {
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              float a0, a1, t0, t1;
              ffma2(a0, a1, __uint_as_float(sr[c4 * 8 + e]), __uint_as_float(sr[c4 * 8 + e + 1]), sl2, sl2,
                    lv[e], lv[e + 1]);
              pr[e] = ex2_approx(a0);
              pr[e + 1] = ex2_approx(a1);
              fadd2(t0, t1, __uint_as_float(dr[c4 * 8 + e]), __uint_as_float(dr[c4 * 8 + e + 1]), dv[e], dv[e + 1]);
              ffma2(ds[e], ds[e + 1], pr[e], pr[e + 1], t0, t1, 0.f, 0.f);
            }
          } else if (JOB == kJobBand || (JOB == kJobBandX && qt.src == 0 && !p.local_bias)) {
            // band boundary tile: the packed steps of the interior, then pairs outside
            // the band (offset outside [lo, lo + span), one unsigned compare each; a
            // padded key has span 0) give p = 0
            const int lo = p.causal ? 0 : -u.r;
            const unsigned span = key_valid ? (unsigned)(p.causal ? u.r + 1 : 2 * u.r + 1) : 0u;
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              const int off = d0 + c * 8 + e;
              float a0, a1, t0, t1;
              ffma2(a0, a1, __uint_as_float(sr[c4 * 8 + e]), __uint_as_float(sr[c4 * 8 + e + 1]), sl2, sl2,
                    lv[e], lv[e + 1]);
              pr[e] = ((unsigned)(off - lo) < span) ? ex2_approx(a0) : 0.f;
              pr[e + 1] = ((unsigned)(off + 1 - lo) < span) ? ex2_approx(a1) : 0.f;
              fadd2(t0, t1, __uint_as_float(dr[c4 * 8 + e]), __uint_as_float(dr[c4 * 8 + e + 1]), dv[e], dv[e + 1]);
              ffma2(ds[e], ds[e + 1], pr[e], pr[e + 1], t0, t1, 0.f, 0.f);
            }
          } else if (JOB == kJobBandX && qt.src == 0) {
            // band query tile with the local bias: pairs inside the band, each with the
            // bias of its offset for query rows that are not global (staged flag)
            const int lo = p.causal ? 0 : -u.r;
            const unsigned span = key_valid ? (unsigned)(p.causal ? u.r + 1 : 2 * u.r + 1) : 0u;
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              const int off = d0 + c * 8 + e;
              const bool in0 = (unsigned)(off - lo) < span, in1 = (unsigned)(off + 1 - lo) < span;
              float b0 = 0.f, b1 = 0.f;
              if (lrow) {
                b0 = (in0 && stgi[kQT + c * 8 + e]) ? __ldg(lrow - u.d * off) : 0.f;
                b1 = (in1 && stgi[kQT + c * 8 + e + 1]) ? __ldg(lrow - u.d * (off + 1)) : 0.f;
              }
              float a0, a1, t0, t1;
              ffma2(a0, a1, b0, b1, kBLog2e, kBLog2e, lv[e], lv[e + 1]);
              ffma2(a0, a1, __uint_as_float(sr[c4 * 8 + e]), __uint_as_float(sr[c4 * 8 + e + 1]), sl2, sl2, a0, a1);
              pr[e] = in0 ? ex2_approx(a0) : 0.f;
              pr[e + 1] = in1 ? ex2_approx(a1) : 0.f;
              fadd2(t0, t1, __uint_as_float(dr[c4 * 8 + e]), __uint_as_float(dr[c4 * 8 + e + 1]), dv[e], dv[e + 1]);
              ffma2(ds[e], ds[e + 1], pr[e], pr[e + 1], t0, t1, 0.f, 0.f);
            }
          } else if (((JOB == kJobBandX && qt.src != 0) || JOB == kJobGlobalKeys || JOB == kJobRandom) &&
                     !p.causal && (JOB == kJobRandom || (u.d & (u.d - 1)) == 0)) {
            // query rows whose window misses the key (global query rows of the band job,
            // the global-key job, the random job): on the staged query position,
            // (unsigned)(qpos - kpos + rd) > 2 rd, or with a power-of-two dilation a query
            // of another residue class.  Rows that do not count have -lse = -inf and give
            // p = 0 by themselves.
            const bool kok = key_valid && !(JOB == kJobGlobalKeys && key_in_rand);
            const int kr = rd - kpos;
            const unsigned span2 = 2u * (unsigned)rd;
            const unsigned dm = JOB == kJobRandom ? 0u : (unsigned)u.d - 1u;
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              float a0, a1, t0, t1;
              ffma2(a0, a1, __uint_as_float(sr[c4 * 8 + e]), __uint_as_float(sr[c4 * 8 + e + 1]), sl2, sl2,
                    lv[e], lv[e + 1]);
              const unsigned x0 = (unsigned)(stgi[c * 8 + e] + kr), x1 = (unsigned)(stgi[c * 8 + e + 1] + kr);
              pr[e] = (kok && (x0 > span2 || (x0 & dm) != 0u)) ? ex2_approx(a0) : 0.f;
              pr[e + 1] = (kok && (x1 > span2 || (x1 & dm) != 0u)) ? ex2_approx(a1) : 0.f;
              fadd2(t0, t1, __uint_as_float(dr[c4 * 8 + e]), __uint_as_float(dr[c4 * 8 + e + 1]), dv[e], dv[e + 1]);
              ffma2(ds[e], ds[e + 1], pr[e], pr[e + 1], t0, t1, 0.f, 0.f);
            }
          } else if (JOB == kJobSide) {
            // side tile: every valid query row, with the side bias of its query block
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              float b0 = 0.f, b1 = 0.f;
              if (sbias) {
                b0 = __ldg(sbias - stgi[kQT + c * 8 + e]);
                b1 = __ldg(sbias - stgi[kQT + c * 8 + e + 1]);
              }
              float a0, a1, t0, t1;
              ffma2(a0, a1, b0, b1, kBLog2e, kBLog2e, lv[e], lv[e + 1]);
              ffma2(a0, a1, __uint_as_float(sr[c4 * 8 + e]), __uint_as_float(sr[c4 * 8 + e + 1]), sl2, sl2, a0, a1);
              pr[e] = key_valid ? ex2_approx(a0) : 0.f;
              pr[e + 1] = key_valid ? ex2_approx(a1) : 0.f;
              fadd2(t0, t1, __uint_as_float(dr[c4 * 8 + e]), __uint_as_float(dr[c4 * 8 + e + 1]), dv[e], dv[e + 1]);
              ffma2(ds[e], ds[e + 1], pr[e], pr[e + 1], t0, t1, 0.f, 0.f);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              bool allowed;
              float b2 = 0.f;
              if (JOB == kJobBand || (JOB == kJobBandX && qt.src == 0)) {
                const int off = d0 + c * 8 + e;
                const bool inband = p.causal ? (off >= 0 && off <= u.r) : (off >= -u.r && off <= u.r);
                allowed = key_valid && inband;
                if (JOB == kJobBandX && lrow && allowed && stgi[kQT + c * 8 + e])
                  b2 = __ldg(lrow - u.d * off) * kBLog2e;
              } else if (JOB == kJobBandX) {
                // a global query row: keys outside its window (inside it the band tile counts)
                allowed = key_valid && !in_window(stgi[c * 8 + e], kpos, rd, u.d, p.causal);
              } else if (JOB == kJobGlobalKeys) {
                allowed = key_valid && !key_in_rand && !in_window(stgi[c * 8 + e], kpos, rd, u.d, p.causal);
              } else if (JOB == kJobSide) {
                allowed = key_valid;
                if (sbias) b2 = __ldg(sbias - stgi[kQT + c * 8 + e]) * kBLog2e;
              } else {
                allowed = key_valid && !in_window(stgi[c * 8 + e], kpos, rd, 1, p.causal);
              }
              pr[e] = allowed ? ex2_approx(__uint_as_float(sr[c4 * 8 + e]) * sl2 + b2 + lv[e]) : 0.f;
              ds[e] = pr[e] * (__uint_as_float(dr[c4 * 8 + e]) + dv[e]);
            }
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            pk[c4 * 4 + e] = pack_bf16x2(pr[2 * e], pr[2 * e + 1]);
            dk[c4 * 4 + e] = pack_bf16x2(ds[2 * e], ds[2 * e + 1]);
          }
        }
        // over columns this thread has already read (half 0: S^T 0-15 of 0-31; half 1:
        // 16-31, read in half 0); the loads of half 1 read columns 32-63
        tmem_st16(lane_base + 128 * g + 16 * half, pk);
        tmem_st16(lane_base + 128 * g + 64 + 16 * half, dk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[g]);
    }
    // epilogue: group 0 writes dV, group 1 writes dK = scale * (dS^T Q), fp32.  Band and
    // side jobs overwrite (padded keys get zeros); the global-key and random jobs add
    // to the rows the band pass wrote.  The TMEM loads are warp-wide, so every thread
    // issues them.
    if (ok && T > 0) ok = mbar_wait_bounded(acc_full, 0, abort_v, kWaitLimitNs);
    if (ok) {
      tc_fence_after();
      constexpr bool kAdd = JOB == kJobGlobalKeys || JOB == kJobRandom;
      size_t prw = 0;
      float* base = g ? p.dk : p.dv;
      bool write = row < u.rows;
      if (JOB == kJobSide) {
        base = g ? p.dsk : p.dsv;
        prw = ((size_t)u.b * p.Hkv + u.hk) * p.S + uk;
      } else if (kAdd) {
        write = key_valid;
        prw = ((size_t)u.b * p.Hkv + u.hk) * p.n + kpos;
      } else if (write) {
        prw = pos_row(p, u, u.hk, p.Hkv, uk);
      }
      float* dst = base + prw * D;
      const float mul = g ? p.scale : 1.f;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t rr[32];
        if (T > 0) {
          tmem_ld32(lane_base + (g ? C::kAccK : C::kAccV) + ch * 32, rr);
          tmem_wait_ld_dep(rr);
        }
        if (write) {
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (T > 0 && key_valid)
              v4 = make_float4(__uint_as_float(rr[q4 * 4]) * mul, __uint_as_float(rr[q4 * 4 + 1]) * mul,
                               __uint_as_float(rr[q4 * 4 + 2]) * mul, __uint_as_float(rr[q4 * 4 + 3]) * mul);
            float4* d4 = reinterpret_cast<float4*>(dst) + ch * 8 + q4;
            if (kAdd) {
              const float4 o = *d4;
              v4 = make_float4(o.x + v4.x, o.y + v4.y, o.z + v4.z, o.w + v4.w);
            }
            *d4 = v4;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (abort_flag) {
    if (tid == 0) {
      atomicOr(p.err, kDevErrTimeout);
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < 2000000ull) {
      }
    }
    __syncthreads();
  }
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Every dQ and dK/dV launch follows the Delta pass (and the gather) of the same
// backward, so it is a programmatic dependent launch: scheduled while the kernel
// before it drains, it sets up its barriers and TMEM and then waits for it.
template <typename K>
cudaError_t launch_kern(K kern, uint32_t smem, int grid, int threads, const BwdParams& p, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (grid <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

cudaError_t launch_bwd_delta(const BwdParams& p, cudaStream_t s) {
  const size_t rows = (size_t)p.B * p.Hq * p.n;
  const size_t warps = (rows + 1) / 2;
  const int blocks = (int)((warps * 32 + 255) / 256);
  if (p.D == 128) bwd_delta_kernel<128><<<blocks, 256, 0, s>>>(p);
  else bwd_delta_kernel<64><<<blocks, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dq(const BwdParams& p, cudaStream_t s) {
  const int grid = min(p.max_qtiles * p.B * p.Hq, p.num_sms);       // persistent
  if (p.extras)
    return p.D == 64 ? launch_kern(bwd_dq_kernel<64, true, false>, BCfg<64>::kSmemBytes, grid, kBThreads, p, s)
                     : launch_kern(bwd_dq_kernel<128, true, false>, BCfg<128>::kSmemBytes, grid, kBThreads, p, s);
  return p.D == 64 ? launch_kern(bwd_dq_kernel<64, false, false>, BCfg<64>::kSmemBytes, grid, kBThreads, p, s)
                   : launch_kern(bwd_dq_kernel<128, false, false>, BCfg<128>::kSmemBytes, grid, kBThreads, p, s);
}

cudaError_t launch_bwd_dq_global_rows(const BwdParams& p, cudaStream_t s) {
  if (p.g == 0) return cudaSuccess;
  const int grid = min(p.B * p.Hq * (p.gpad / kTile), p.num_sms);   // persistent
  return p.D == 64 ? launch_kern(bwd_dq_kernel<64, false, true>, BCfg<64>::kSmemBytes, grid, kBThreads, p, s)
                   : launch_kern(bwd_dq_kernel<128, false, true>, BCfg<128>::kSmemBytes, grid, kBThreads, p, s);
}

template <int JOB>
static cudaError_t launch_dkv_job(const BwdParams& p, int grid, cudaStream_t s) {
  return p.D == 64 ? launch_kern(bwd_dkv_kernel<64, JOB>, KCfg<64>::kSmemBytes, grid, kDkvThreads, p, s)
                   : launch_kern(bwd_dkv_kernel<128, JOB>, KCfg<128>::kSmemBytes, grid, kDkvThreads, p, s);
}

cudaError_t launch_bwd_dkv(const BwdParams& p, cudaStream_t s) {
  const int grid = p.max_ktiles * p.B * p.Hkv;
  return p.extras ? launch_dkv_job<kJobBandX>(p, grid, s) : launch_dkv_job<kJobBand>(p, grid, s);
}

cudaError_t launch_bwd_dkv_global_keys(const BwdParams& p, cudaStream_t s) {
  if (p.g == 0) return cudaSuccess;
  return launch_dkv_job<kJobGlobalKeys>(p, p.B * p.Hkv * (p.gpad / kTile), s);
}

cudaError_t launch_bwd_dkv_side(const BwdParams& p, cudaStream_t s) {
  if (p.S == 0) return cudaSuccess;
  return launch_dkv_job<kJobSide>(p, p.B * p.Hkv * ((p.S + kTile - 1) / kTile), s);
}

cudaError_t launch_bwd_dkv_random(const BwdParams& p, cudaStream_t s) {
  if (!p.rand_blocks || p.num_rand == 0) return cudaSuccess;
  return launch_dkv_job<kJobRandom>(p, p.B * p.Hkv * ((p.n + kTile - 1) / kTile), s);
}

}  // namespace swa
