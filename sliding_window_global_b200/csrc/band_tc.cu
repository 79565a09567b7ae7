// band_tc.cu -- tcgen05 (5th-generation tensor core) kernel for banded sparse
// self-attention on sm_100a: bf16 inputs, fp32 accumulation in TMEM.
//
// A unit of work is a pair of 128-row query tiles (A and B, consecutive rows) of
// one (batch, query head, residue class).  It walks a list of 128-key tiles:
//   band tiles   -- keys of the (dilated, optionally causal) sliding window
//                   ("精读笔记：Big Bird" §3.2.1; the Longformer page §二 for
//                   dilation; SWAN-GPT §3.3(1) for the causal 512-key window); only
//                   the tiles the two windows touch are loaded, so fully masked
//                   tiles are skipped and each K/V tile feeds both query tiles;
//   global tiles -- the gathered global tokens every query also attends to,
//                   minus those already inside its window (BigBird §3.2.3, ITC);
//   side tiles   -- appended side keys with the additive bucketed bias of the
//                   LongT5 Transient-Global attention ("LongT5 长序列模型完全指南",
//                   Transient-Global and 源码级证据 sections);
//   random tiles -- the random key blocks of each query tile (BigBird §3.2.2:
//                   every query also attends to randomly chosen keys), minus keys
//                   inside the row's window; only the tile they belong to uses them.
// Band tiles may carry a local relative-position bias indexed by key - query
// offset (the LongT5 page, 相对位置编码: the local attention's bias is computed
// once over the window); its row for the unit's head is staged in shared memory.
// With dilation d a query at position c + d*u only meets keys c + d*u', so each
// residue class is a plain band of radius r over rows c, c+d, ..., loaded through
// strided TMA tensor maps.
//
// The kernel is persistent: one CTA per SM walks units (query heads fastest, so
// CTAs running together share K/V tiles through L2).  TMEM, barriers and the
// K/V ring live across units, the next unit's Q tiles are fetched while the
// current unit finishes, and the epilogue stores O straight from registers.
//
// MODE 1 computes global query rows (full attention over all valid keys plus side
// keys), split over key ranges into fp32 partials that a logsumexp merge
// combines; tile B is unused there.
//
// Warp roles (384 threads; the control warpgroup gives registers to the softmax
// warpgroups with setmaxnreg):
//   warps 0-3   softmax of tile A, warps 4-7 softmax of tile B: thread t of the
//               group owns query row t (TMEM lane t).  Per key tile: load S from
//               TMEM, mask (boundary tiles only), scale, add bias (side tiles;
//               band tiles with a local bias),
//               running max m / sum l with a lazy O rescale (only when the max
//               grows by more than 2^8), exponentiate -- part of the elements on
//               the MUFU unit, part with a polynomial on the FMA pipe -- and write
//               P (bf16) back into the TMEM columns of S.  Epilogue: O / l.
//   warp 8      TMA producer: Q tiles, then K/V tiles into an NS-stage ring.
//   warp 9      TMEM allocator and MMA issuer.  P over S (D = 128): it issues
//               both tiles' MMAs; per key tile j, for A then B, O += P(j) V(j)
//               (P read from TMEM) immediately followed by S = Q K(j+1)^T into
//               the same TMEM columns, so the tensor core works on one query
//               tile while the other one's softmax runs.  MMAs from one thread
//               execute in order, so a new S never overwrites a P that an
//               earlier MMA still reads.  Separate P (D = 64): warp 9 issues
//               tile A's MMAs and warp 10 tile B's, each the next S of its tile
//               as soon as the softmax has read the current one; the two
//               issuers share only the K/V ring (read-only) and release each
//               slot together.  Other warps of the group idle.
#include "ptx.cuh"
#include "side_mean.cuh"
#include "softmax_math.cuh"
#include "swa_kernels.h"

namespace swa {
namespace {

constexpr int kSoftmaxThreads = 256;
constexpr int kThreads = 384;                 // 3 warpgroups: softmax A, softmax B, control
// Registers per thread after reallocation, per head size: the softmax warps get 200
// at D = 128 and 216 at D = 64, the control warps 104 and 72 (256 * 200 + 128 * 104 =
// 256 * 216 + 128 * 72 = 384 * 168, the budget the CTA is launched with).  The split
// was chosen by the compiler's spill counts: at D = 64 the wider softmax budget
// removes most spills, at D = 128 the control warps need the 104.
template <int D>
__host__ __device__ constexpr int regs_softmax() {
  return D == 64 ? 216 : 200;
}
template <int D>
__host__ __device__ constexpr int regs_control() {
  return D == 64 ? 72 : 104;
}
constexpr uint32_t kSub = 128 * 128;          // one 128-row x 128-byte swizzle sub-tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;     // log2 units

#ifndef SWA_EMU_PER32_D128
#define SWA_EMU_PER32_D128 0
#endif
#ifndef SWA_EMU_PER32_D64
#define SWA_EMU_PER32_D64 8
#endif
// Of every 32 exponentials, this many (a multiple of 4) are evaluated by the
// FMA-pipe polynomial instead of MUFU.EX2; measured best per head size.
template <int D>
__host__ __device__ constexpr int emu_per32() {
  return D == 128 ? SWA_EMU_PER32_D128 : SWA_EMU_PER32_D64;
}

// Where the tile max is taken: once after the tile-kind branches (D = 128), or
// inside each branch (D = 64).  Both compute the same value; the code placement
// was measured faster for each head size.
template <int D>
__host__ __device__ constexpr bool max_after_branches() {
  return D == 128;
}

template <int D>
struct Cfg {
  static constexpr int NS = (D == 64) ? 4 : 2;                 // K/V ring stages
  static constexpr uint32_t kTileBytes = 128u * D * 2u;        // one 128 x D bf16 tile
  static constexpr uint32_t kQOff = 0;                         // Q_A, Q_B
  static constexpr uint32_t kKOff = 2 * kTileBytes;
  static constexpr uint32_t kVOff = kKOff + NS * kTileBytes;
  static constexpr uint32_t kBiasOff = kVOff + NS * kTileBytes;  // 4 shifted copies
  static constexpr uint32_t kBarOff = kBiasOff + 4 * kBiasCopy * 4;
  static constexpr int kNumBars = 2 + 2 + 3 * NS + 2 + 2 + 2 + 2 + 2 + 2;
  static constexpr uint32_t kSmemBytes = kBarOff + kNumBars * 8 + 1024;
  // TMEM columns.  D = 128: S_A | S_B | O_A | O_B, P written over S.  D = 64 has
  // room for separate P buffers (S_A | S_B | P_A | P_B | O_A | O_B), so the next
  // S can be computed while the softmax of the current one still runs.
  static constexpr bool kSepP = (D == 64);
  static constexpr uint32_t kTmemCols = 512;
  __host__ __device__ static constexpr uint32_t s_col(int x) { return x ? 128u : 0u; }
  __host__ __device__ static constexpr uint32_t p_col(int x) { return kSepP ? 256u + 64u * x : s_col(x); }
  __host__ __device__ static constexpr uint32_t o_col(int x) {
    return kSepP ? 384u + 64u * x : 256u + (x ? D : 0);
  }
};

// The register split must fit the budget the CTA is launched with (a larger sum
// would leave setmaxnreg.inc waiting), and the shared memory one CTA per SM.
// setmaxnreg moves registers only between the warps of one SM sub-partition (warp
// w runs on sub-partition w % 4), so the split must also fit each sub-partition's
// share: here one warp of each softmax group and one control warp.
template <int D>
constexpr bool split_fits() {
  return kSoftmaxThreads * regs_softmax<D>() + (kThreads - kSoftmaxThreads) * regs_control<D>() <= kThreads * 168 &&
         2 * regs_softmax<D>() + regs_control<D>() <= 3 * 168;
}
static_assert(kThreads == 12 * 32 && kSoftmaxThreads == 8 * 32 && split_fits<64>() && split_fits<128>(),
              "setmaxnreg split exceeds the launch budget or a sub-partition's registers");
static_assert(Cfg<64>::kSmemBytes + 2 * kTile * 4 + 16 <= 227 * 1024, "shared memory, D = 64");
static_assert(Cfg<128>::kSmemBytes + 2 * kTile * 4 + 16 <= 227 * 1024, "shared memory, D = 128");
static_assert(emu_per32<64>() % 4 == 0 && emu_per32<64>() <= 32 && emu_per32<128>() % 4 == 0 &&
                  emu_per32<128>() <= 32,
              "polynomial exponentials come in groups of four");

// ------------------------------------------------------------------ work description
struct Work {
  bool valid;           // the unit id names real work
  int b, h, hk, cls, d, c, r;
  int hx[2];            // query head of tile A, B (equal unless heads are paired)
  int u0[2];            // first row (class coordinates / global slot) of tile A, B
  int rows[2];          // rows that exist
  int nvalid[2];        // rows below the valid length / below g
  int Vc;               // valid rows of the class (MODE 0) / valid keys (MODE 1)
  int split;            // MODE 1 key split
  bool active[2];
  int band_lo;          // first key of band tile 0
  int nband, ngc, nside, total;
  int rand0;            // first random tile; with both tiles active they alternate A, B, A, ...
  int nrand[2];         // random tiles of tile A, B (equal when both are active)
  int key_end;          // MODE 1: keys at or beyond this are masked
  int lo[2], hi[2];     // band key range of each query tile (class coordinates)
};

template <int MODE>
__device__ __forceinline__ int total_units(const AttnParams& p) {
  return MODE == 0 ? p.max_units * p.B * (p.pair_heads ? p.Hq / 2 : p.Hq)
                   : p.nsplit * (p.gpad / kTile) * p.B * p.Hq;
}

template <int MODE, bool RAND>
__device__ __forceinline__ void decode_work(const AttnParams& p, int unit_id, Work& w) {
  if (MODE == 0) {
    // unit ids run over (unit, batch, head or head pair), heads fastest
    const int hunits = p.pair_heads ? p.Hq / 2 : p.Hq;
    const int BH = p.B * hunits;
    const int bh = unit_id % BH;
    int unit = unit_id / BH;
    w.b = bh / hunits;
    w.h = p.pair_heads ? 2 * (bh % hunits) : bh % hunits;
    w.hx[0] = w.h;
    w.hx[1] = p.pair_heads ? w.h + 1 : w.h;
    w.valid = unit < p.tiles[w.h];
    w.hk = w.h / p.G;
    w.r = p.window[w.h];
    const int base = p.class_base[w.h];
    w.d = p.cls[base].d;
    const int nres = p.cls[base].nres;
    const int per_unit = p.pair_heads ? 1 : 2;           // row tiles per unit and class
    int c = 0;
    for (; c < nres - 1; ++c) {
      const int tc = (p.cls[base + c].n_c + kTile - 1) / kTile;
      const int uc = (tc + per_unit - 1) / per_unit;
      if (unit < uc) break;
      unit -= uc;
    }
    w.c = c;
    w.cls = base + c;
    const int nc = p.cls[w.cls].n_c;
    int V = p.valid_len ? p.valid_len[w.b] : p.n;
    V = min(V, p.n);
    w.Vc = V > c ? (V - c + w.d - 1) / w.d : 0;
    w.split = 0;
    w.key_end = 0;
    for (int x = 0; x < 2; ++x) {
      w.u0[x] = p.pair_heads ? unit * kTile : unit * 2 * kTile + x * kTile;
      w.rows[x] = w.valid ? max(0, min(kTile, nc - w.u0[x])) : 0;
      w.nvalid[x] = max(0, min(w.rows[x], w.Vc - w.u0[x]));
      w.active[x] = w.nvalid[x] > 0;
      w.lo[x] = max(0, w.u0[x] - w.r);
      const int last = w.u0[x] + w.nvalid[x] - 1;
      w.hi[x] = p.causal ? min(w.Vc, last + 1) : min(w.Vc, last + w.r + 1);
    }
    w.band_lo = w.lo[0];
    const int hi = w.active[1] ? max(w.hi[0], w.hi[1]) : w.hi[0];
    w.nband = w.active[0] ? (hi - w.band_lo + kTile - 1) / kTile : 0;
    w.ngc = (w.active[0] && p.g > 0) ? (p.g + kTile - 1) / kTile : 0;
    w.nside = (w.active[0] && p.S > 0) ? (p.S + kTile - 1) / kTile : 0;
  } else {
    w.valid = true;
    w.split = unit_id % p.nsplit;
    const int rest = unit_id / p.nsplit;
    const int gtiles = p.gpad / kTile;
    const int gt = rest % gtiles;
    const int bh = rest / gtiles;
    w.b = bh / p.Hq;
    w.h = bh % p.Hq;
    w.hx[0] = w.hx[1] = w.h;
    w.hk = w.h / p.G;
    w.r = 0;
    w.d = 1;
    w.c = 0;
    w.cls = p.dense_class;
    int V = p.valid_len ? p.valid_len[w.b] : p.n;
    V = min(V, p.n);
    w.Vc = V;
    w.u0[0] = gt * kTile;
    w.rows[0] = min(kTile, p.gpad - w.u0[0]);
    w.nvalid[0] = max(0, min(w.rows[0], p.g - w.u0[0]));
    w.u0[1] = 0;
    w.rows[1] = w.nvalid[1] = 0;
    w.active[1] = false;
    w.ngc = 0;
    if (w.split < p.nsplit_keys) {
      const int k0 = w.split * p.split_keys;
      const int k1 = min(V, k0 + p.split_keys);
      w.band_lo = k0;
      w.key_end = k1;
      w.nband = (k1 > k0) ? (k1 - k0 + kTile - 1) / kTile : 0;
      w.nside = 0;
    } else {
      w.band_lo = 0;
      w.key_end = 0;
      w.nband = 0;
      w.nside = (p.S + kTile - 1) / kTile;
    }
    w.active[0] = w.nvalid[0] > 0 && (w.nband + w.nside) > 0;
    if (!w.active[0]) w.nband = w.nside = 0;
    w.lo[0] = w.band_lo;
    w.hi[0] = w.key_end;
    w.lo[1] = w.hi[1] = 0;
  }
  w.rand0 = w.nband + w.ngc + w.nside;
  w.nrand[0] = (RAND && MODE == 0 && w.active[0]) ? p.num_rand : 0;
  w.nrand[1] = (RAND && MODE == 0 && w.active[1]) ? p.num_rand : 0;
  w.total = w.rand0 + w.nrand[0] + w.nrand[1];
}

// Owner (query tile) and index t of random tile j >= w.rand0.  Alternating the two
// tiles' random blocks lets one tile's softmax overlap the other tile's MMAs.
__device__ __forceinline__ int rand_owner(const Work& w, int j, int& t) {
  const int k = j - w.rand0;
  if (w.nrand[1] > 0 && w.nrand[0] > 0) {
    t = k >> 1;
    return k & 1;
  }
  t = k;
  return w.nrand[0] > 0 ? 0 : 1;
}

// Random key block t of query tile x (query block u0 / kTile; dilation 1 only).
__device__ __forceinline__ int rand_block(const AttnParams& p, int b, int head, int u0, int t) {
  const int nqb = (p.n + kTile - 1) / kTile;
  return __ldg(p.rand_blocks + (((size_t)b * p.Hq + head) * nqb + u0 / kTile) * p.num_rand + t);
}

// The fields of one query tile as scalars: the softmax warps pick their tile at
// run time, and indexing Work's two-element arrays with a run-time index would
// put the whole struct in local memory.
struct TileRows {
  int u0, rows, nvalid, lo, hi, head;
  bool active;
};

__device__ __forceinline__ TileRows tile_rows(const Work& w, int x) {
  TileRows t;
  t.u0 = x ? w.u0[1] : w.u0[0];
  t.rows = x ? w.rows[1] : w.rows[0];
  t.nvalid = x ? w.nvalid[1] : w.nvalid[0];
  t.lo = x ? w.lo[1] : w.lo[0];
  t.hi = x ? w.hi[1] : w.hi[0];
  t.head = x ? w.hx[1] : w.hx[0];
  t.active = x ? w.active[1] : w.active[0];
  return t;
}

// Does query tile x (fields t) use key tile j?
__device__ __forceinline__ bool uses(const Work& w, const TileRows& t, int x, int j) {
  if (!t.active || j < 0 || j >= w.total) return false;
  if (j >= w.rand0) {                                   // a tile's own random blocks
    int t;
    return rand_owner(w, j, t) == x;
  }
  if (j >= w.nband) return true;                        // global and side tiles: every row
  const int kv0 = w.band_lo + j * kTile;
  return kv0 < t.hi && kv0 + kTile > t.lo;
}

__device__ __forceinline__ void tile_source(const AttnParams& p, const Work& w, int j,
                                            const CUtensorMap*& mk, const CUtensorMap*& mv,
                                            int& y) {
  if (j < w.nband) {
    mk = &p.mk[w.cls];
    mv = &p.mv[w.cls];
    y = w.band_lo + j * kTile;
  } else if (j < w.nband + w.ngc) {
    mk = &p.mgk;
    mv = &p.mgv;
    y = (j - w.nband) * kTile;
  } else if (j < w.rand0) {
    mk = &p.msk;
    mv = &p.msv;
    y = (j - w.nband - w.ngc) * kTile;
  } else {
    // random key block (dilation 1: the class map is the plain key sequence)
    int t;
    const int x = rand_owner(w, j, t);
    mk = &p.mk[w.cls];
    mv = &p.mv[w.cls];
    y = rand_block(p, w.b, x ? w.hx[1] : w.hx[0], x ? w.u0[1] : w.u0[0], t) * kTile;
  }
}

template <int D>
__device__ __forceinline__ void tma_tile(void* dst, const CUtensorMap* map, uint64_t* bar, int y,
                                         int z) {
  tma_load_3d(dst, map, bar, 0, y, z);
  if (D == 128) tma_load_3d(static_cast<uint8_t*>(dst) + kSub, map, bar, 64, y, z);
}

// Row max of 128 values: 8 independent chains of 3-input maxima, then a tree.
__device__ __forceinline__ float row_max128(const float (&x)[kTile]) {
  float m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = fmaxf(x[i], x[8 + i]);
#pragma unroll
  for (int e = 16; e < kTile; e += 16) {
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fmax3(m[i], x[e + i], x[e + 8 + i]);
  }
  return fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// ------------------------------------------------------------------ output rows
__device__ __forceinline__ size_t out_row(const AttnParams& p, const Work& w, const TileRows& t,
                                          int row) {
  const int pos = w.c + w.d * (t.u0 + row);
  return (size_t)(w.b * p.Hq + t.head) * p.n + pos;
}

template <int D>
__device__ void write_zero_row(const AttnParams& p, const Work& w, const TileRows& t, int row) {
  if (row >= t.rows || row < t.nvalid) return;
  const size_t off = out_row(p, w, t, row);
  uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + off * D);
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i] = make_uint4(0, 0, 0, 0);
  if (p.lse) p.lse[off] = -INFINITY;
}

template <int D>
__device__ void write_neutral_partial(const AttnParams& p, const Work& w, int row) {
  const int slot = w.u0[0] + row;
  if (row >= kTile || slot >= p.gpad) return;
  const size_t prow = ((size_t)w.split * p.B * p.Hq + (size_t)w.b * p.Hq + w.h) * p.gpad + slot;
  float4* po = reinterpret_cast<float4*>(p.part_o + prow * D);
  for (int i = 0; i < D / 4; ++i) po[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  p.part_lse[prow] = -INFINITY;
}

// Fused Transient-Global prologue (AGG): this CTA's share of the side keys and
// values (16-byte column groups of the side rows of k, then of v), all threads.
template <int D>
__device__ __forceinline__ void side_prologue(const AttnParams& p, int tid, int nthreads) {
  constexpr int VEC = 8;                                   // bf16
  constexpr int groups = D / VEC;
  const long long rows = (long long)p.B * p.Hkv * p.S;     // per tensor
  const long long items = 2 * rows * groups;
  const long long lo = items * blockIdx.x / gridDim.x, hi = items * (blockIdx.x + 1) / gridDim.x;
  for (long long t = lo + tid; t < hi; t += nthreads) {
    const bool is_v = t >= rows * groups;
    const long long u = is_v ? t - rows * groups : t;
    const int cg = (int)(u % groups);
    const long long r = u / groups;
    const int s = (int)(r % p.S);
    const long long bh = r / p.S;
    const int b = (int)(bh / p.Hkv);
    const int V = min(p.valid_len ? __ldg(p.valid_len + b) : p.n, p.n);
    side_mean_vec<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(is_v ? p.agg_v : p.agg_k),
                                 static_cast<__nv_bfloat16*>(is_v ? p.agg_sv : p.agg_sk), (size_t)bh, s, cg,
                                 p.n, D, p.side_block, V);
  }
}

// LOCAL: band tiles carry the local relative-position bias; RAND: query tiles have
// random key blocks (MODE 0 only); AGG: the CTAs first build the side keys / values
// from k and v (cooperative launch) and load side tiles once every CTA has counted
// itself done; GLOB: the tile lists hold global-column tiles (launches with global
// tokens).  They are template parameters so that kernels without them keep their
// register schedule.
template <int D, int MODE, bool LOCAL, bool RAND, bool AGG, bool GLOB>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ AttnParams p) {
  using C = Cfg<D>;
  constexpr int NS = C::NS;
  constexpr bool kMaxAfter = max_after_branches<D>();
  constexpr int kIssuers = C::kSepP ? 2 : 1;              // MMA-issuing warps
  constexpr int kTilesPerIssuer = 2 / kIssuers;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::kQOff;
  uint8_t* sK = smem + C::kKOff;
  uint8_t* sV = smem + C::kVOff;
  float* sBias = reinterpret_cast<float*>(smem + C::kBiasOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* q_full = bars;                // [2]
  uint64_t* q_empty = bars + 2;           // [2]
  uint64_t* k_full = bars + 4;            // [NS]
  uint64_t* v_full = k_full + NS;
  uint64_t* kv_empty = v_full + NS;
  uint64_t* s_full = kv_empty + NS;       // [2]
  uint64_t* p_full = s_full + 2;          // [2]
  uint64_t* o_full = p_full + 2;          // [2]
  uint64_t* s_free = o_full + 2;          // [2] S read into registers (separate-P layout)
  uint64_t* pv_done = s_free + 2;         // [2] a PV finished: P buffer free, O updated
  uint64_t* p_half = pv_done + 2;         // [2] P of keys 0-63 written (P-over-S layout)
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ __align__(16) int sGpos[2 * kTile];   // the current global tile's keys, per group

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int nunits = total_units<MODE>(p);
  const bool has_bias = p.bias && p.S > 0;
  constexpr bool has_local = LOCAL && MODE == 0;
  // shared bias area: 4 copies of the local-bias row (stride lstride floats), then
  // 4 copies of the side-bias segment (stride side_stride)
  const int lstride = has_local ? p.local_stride : 0;
  const int side_stride = kBiasCopy - lstride;
  float* sLocal = sBias;
  float* sSide = sBias + 4 * lstride;

  if (tid == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(&q_full[x], 1);
      mbar_init(&q_empty[x], 1);
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], kTile);
      mbar_init(&o_full[x], 1);
      mbar_init(&s_free[x], kTile);
      mbar_init(&pv_done[x], 1);
      mbar_init(&p_half[x], kTile);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], kIssuers);    // released by every MMA issuer
    }
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
  // Launched right behind the kernel before it, this kernel has set up its barriers
  // and TMEM meanwhile; nothing before this point reads global memory.  The band
  // kernel (MODE 0) waits here for the gathered global rows, then lets the
  // global-row kernel after it start on SMs its CTAs leave: that kernel reads only
  // the gathered rows, which are complete now, and waits for this grid only at its
  // end, before the merge that overwrites the band's global rows.
  if (MODE == 0) {
    grid_dependency_wait();
    if (GLOB) grid_launch_dependents();
  }
  if (AGG) {
    side_prologue<D>(p, tid, kThreads);
    fence_proxy_async_global();                // side rows written here are read by TMA
    __threadfence();
    __syncthreads();
    if (tid == 0) atomicAdd(p.agg_count, 1u);  // after the whole CTA's stores
  }
  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    setmaxnreg_dec<regs_control<D>()>();
    if (lane == 0) {
      int qloads[2] = {0, 0};
      int kv = 0;                                   // K/V tiles loaded so far (ring position)
      bool ok = true;
      bool side_ready = false;                      // AGG: every CTA counted
      for (int uid = blockIdx.x; ok && uid < nunits; uid += gridDim.x) {
        Work w;
        decode_work<MODE, RAND>(p, uid, w);
        if (!w.active[0]) continue;
        const CUtensorMap* mq = (MODE == 0) ? &p.mq[w.cls] : &p.mgq;
        const int kz = w.b * p.Hkv + w.hk;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          if (!ok) break;
          const int qz = w.b * p.Hq + w.hx[x];
          if (!w.active[x]) continue;
          if (qloads[x] > 0 &&
              !mbar_wait_bounded(&q_empty[x], (qloads[x] - 1) & 1, abort_v, kWaitLimitNs)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&q_full[x], C::kTileBytes);
          tma_tile<D>(sQ + x * C::kTileBytes, mq, &q_full[x], w.u0[x], qz);
          ++qloads[x];
        }
        for (int j = 0; ok && j < w.total; ++j, ++kv) {
          const int st = kv % NS;
          const int use = kv / NS;
          if (kv >= NS && !mbar_wait_bounded(&kv_empty[st], (use - 1) & 1, abort_v, kWaitLimitNs)) {
            ok = false;
            break;
          }
          if (AGG && !side_ready && j >= w.nband + w.ngc && j < w.rand0) {
            // first side tile of this CTA: every CTA must have built its share
            if (!wait_count_bounded(p.agg_count, gridDim.x, abort_v, kWaitLimitNs)) {
              ok = false;
              break;
            }
            side_ready = true;
          }
          const CUtensorMap *mk, *mv;
          int y;
          tile_source(p, w, j, mk, mv, y);
          mbar_arrive_expect_tx(&k_full[st], C::kTileBytes);
          tma_tile<D>(sK + st * C::kTileBytes, mk, &k_full[st], y, kz);
          mbar_arrive_expect_tx(&v_full[st], C::kTileBytes);
          tma_tile<D>(sV + st * C::kTileBytes, mv, &v_full[st], y, kz);
        }
      }
    }
  } else if (warp == 9 || (kIssuers == 2 && warp == 10)) {
    // ------------------------------------------------------------ MMA issuers
    // P over S (D = 128): warp 9 issues both tiles' MMAs in one fixed order, which
    // keeps the two softmax groups half a period apart.  Separate P (D = 64): warp
    // 9 issues tile A's MMAs and warp 10 tile B's, so neither tile's products wait
    // behind the other tile's barriers.
    setmaxnreg_dec<regs_control<D>()>();
    if (lane == 0) {
      const int x0 = (kIssuers == 2) ? warp - 9 : 0;   // first tile of this issuer
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
      // low descriptor words of tile buffer 0 / ring slot 0 (128-byte swizzle; V is
      // read MN-major, its 64-column sub-tiles kSub apart); products add offsets
      const uint32_t q_lo = sdesc_lo(smem_u32(sQ), 16);
      const uint32_t k_lo = sdesc_lo(smem_u32(sK), 16);
      const uint32_t v_lo = sdesc_lo(smem_u32(sV), kSub);
      int qwaits[kTilesPerIssuer] = {}, pwaits[kTilesPerIssuer] = {};
      int nqk[kTilesPerIssuer] = {};                    // QKs issued per tile buffer (kernel-wide)
      int kv = 0;
      bool ok = true;
      for (int uid = blockIdx.x; ok && uid < nunits; uid += gridDim.x) {
        Work w;
        decode_work<MODE, RAND>(p, uid, w);
        if (!w.active[0]) continue;
        const int T = w.total;
        // the tiles' fields as scalars (x0 is a run-time value with two issuers)
        TileRows tr[kTilesPerIssuer];
        int first[kTilesPerIssuer], last[kTilesPerIssuer], issued[kTilesPerIssuer], npv[kTilesPerIssuer];
#pragma unroll
        for (int i = 0; i < kTilesPerIssuer; ++i) {
          tr[i] = tile_rows(w, x0 + i);
          first[i] = last[i] = issued[i] = -1;
          npv[i] = 0;
          for (int j = 0; j < T; ++j)
            if (uses(w, tr[i], x0 + i, j)) {
              if (first[i] < 0) first[i] = j;
              last[i] = j;
            }
        }
        auto issue_qk = [&](int i, int j) -> bool {
          const int x = x0 + i;
          const int g = kv + j;
          if (!mbar_wait_bounded(&k_full[g % NS], (g / NS) & 1, abort_v, kWaitLimitNs)) return false;
          // separate-P layout: S_x is rewritten only after the softmax read the last one
          if (C::kSepP && nqk[i] > 0 &&
              !mbar_wait_bounded(&s_free[x], (nqk[i] - 1) & 1, abort_v, kWaitLimitNs))
            return false;
          ++nqk[i];
          tc_fence_after();
          const uint32_t qd = q_lo + x * (C::kTileBytes >> 4);
          const uint32_t kd = k_lo + (g % NS) * (C::kTileBytes >> 4);
          const uint32_t sd = tmem + C::s_col(x);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * kSub + (kk & 3) * 32) >> 4;
            umma_ss_lo(sd, qd + off, kd + off, idesc_qk, kk > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[x]);
          if (j == last[i]) umma_commit(&q_empty[x]);   // Q_x may be refilled once this QK is done
          issued[i] = j;
          return true;
        };
#pragma unroll
        for (int i = 0; i < kTilesPerIssuer; ++i) {
          if (!ok) break;
          if (!tr[i].active) continue;
          ok = mbar_wait_bounded(&q_full[x0 + i], qwaits[i] & 1, abort_v, kWaitLimitNs);
          ++qwaits[i];
          if (ok) ok = issue_qk(i, first[i]);
        }
        for (int j = 0; ok && j < T; ++j) {
          const int g = kv + j;
          const int st = g % NS;
          bool any = false;                           // this issuer reads the slot of tile j
#pragma unroll
          for (int i = 0; i < kTilesPerIssuer; ++i) {
            const bool u = uses(w, tr[i], x0 + i, j);
            any = any || u;
            if (ok && u && issued[i] < j) ok = issue_qk(i, j);
          }
          if (C::kSepP) {
            // the next S of each tile as soon as its softmax has read the current one
            // (its next key tile may be j + 2 when random tiles alternate; a tile up
            // to j + NS - 1 is loadable: its ring slot was freed by tile <= j - 1)
#pragma unroll
            for (int i = 0; i < kTilesPerIssuer; ++i) {
              if (!ok || !uses(w, tr[i], x0 + i, j) || issued[i] != j) continue;
              int jn = j + 1;
              while (jn < T && jn < j + NS && !uses(w, tr[i], x0 + i, jn)) ++jn;
              if (jn < T && jn < j + NS) ok = issue_qk(i, jn);
            }
          }
          if (!ok) break;
          // With two issuers both wait for V of every tile of the unit, used or not,
          // before they release its ring slot: the slot's next load needs both
          // releases, so neither issuer can arrive twice on one phase of kv_empty.
          if (!mbar_wait_bounded(&v_full[st], (g / NS) & 1, abort_v, kWaitLimitNs)) { ok = false; break; }
          if (!any) {
            mbar_arrive(&kv_empty[st]);               // no MMA of this issuer reads the slot
            continue;
          }
          const uint32_t vd = v_lo + st * (C::kTileBytes >> 4);
#pragma unroll
          for (int i = 0; i < kTilesPerIssuer; ++i) {
            const int x = x0 + i;
            if (!ok) break;
            if (!uses(w, tr[i], x, j)) continue;
            if (!C::kSepP) {
              // P over S: the first half of P (keys 0-63) is published early, so the
              // PV over it overlaps the exponentials of the second half
              if (!mbar_wait_bounded(&p_half[x], pwaits[i] & 1, abort_v, kWaitLimitNs)) { ok = false; break; }
              tc_fence_after();
              const uint32_t first = npv[i] > 0 ? 1u : 0u;
#pragma unroll
              for (int kk = 0; kk < kTile / 32; ++kk)
                umma_ts_lo(tmem + C::o_col(x), tmem + C::p_col(x) + kk * 8, vd + ((kk * 2048) >> 4), idesc_pv,
                           kk > 0 ? 1u : first);
            }
            if (!mbar_wait_bounded(&p_full[x], pwaits[i] & 1, abort_v, kWaitLimitNs)) { ok = false; break; }
            ++pwaits[i];
            tc_fence_after();
            const uint32_t first = npv[i] > 0 ? 1u : 0u;
#pragma unroll
            for (int kk = C::kSepP ? 0 : kTile / 32; kk < kTile / 16; ++kk)
              umma_ts_lo(tmem + C::o_col(x), tmem + C::p_col(x) + kk * 8, vd + ((kk * 2048) >> 4), idesc_pv,
                         kk > 0 ? 1u : first);
            ++npv[i];
            if (C::kSepP) umma_commit(&pv_done[x]);
            if (j == last[i]) umma_commit(&o_full[x]);
            else if (!C::kSepP && uses(w, tr[i], x, j + 1)) ok = issue_qk(i, j + 1);
          }
          umma_commit(&kv_empty[st]);
        }
        kv += T;
      }
    }
  } else if (warp >= 10) {
    setmaxnreg_dec<regs_control<D>()>();
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    setmaxnreg_inc<regs_softmax<D>()>();
    const int x = warp >> 2;                   // 0: tile A, 1: tile B
    const int row = tid & 127;                 // TMEM lane == row in the tile
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t s_addr = lane_base + C::s_col(x);
    const uint32_t p_addr = lane_base + C::p_col(x);
    const uint32_t o_addr = lane_base + C::o_col(x);
    int pw = 0;                                // P buffers written (separate-P layout)
    const float sl2 = p.scale_log2;
    int it = 0;                                // S/P tiles handled so far (barrier phase)
    int oc = 0;                                // units finished (o_full phase)
    bool ok = true;
    for (int uid = blockIdx.x; ok && uid < nunits; uid += gridDim.x) {
      Work w;
      decode_work<MODE, RAND>(p, uid, w);
      if (!w.valid) continue;
      const TileRows tr = tile_rows(w, x);
      if (!w.active[0]) {
        if (MODE == 0) write_zero_row<D>(p, w, tr, row);
        else if (x == 0) write_neutral_partial<D>(p, w, row);
        continue;
      }
      const int T = w.total;
      const bool row_valid = row < tr.nvalid;
      const int u = tr.u0 + row;
      int pos = 0;
      if (MODE == 0) pos = w.c + w.d * u;
      else if (row_valid)   // clamped: a broken precondition must not index the bias out of bounds
        pos = min(max(p.global_idx[(size_t)w.b * p.g + w.u0[0] + row], 0), p.n - 1);

      // Bias rows of this unit, four copies shifted by 0..3 floats so that every
      // row can read 16-byte aligned vectors (both groups stage together).
      // Local bias: v[t + r_eff + kLocalPad] = bias of key offset d*t (class
      // coordinates t), zero outside |t| <= r; band tiles read 128 consecutive
      // entries starting anywhere in [-r_eff - 254, r_eff + 127] (r_eff = min(r, n_c)).
      const int r_eff = min(w.r, p.cls[w.cls].n_c);
      int qblk_hi = 0, qblk_lo = 0;
      bool bias_staged = false;
      if (has_bias) {
        int pos_lo, pos_hi;
        if (MODE == 0) {
          const int last_row = w.active[1] ? w.u0[1] + w.nvalid[1] - 1 : w.u0[0] + w.nvalid[0] - 1;
          pos_lo = w.c + w.d * w.u0[0];
          pos_hi = w.c + w.d * last_row;
        } else {
          pos_lo = min(max(p.global_idx[(size_t)w.b * p.g + w.u0[0]], 0), p.n - 1);
          pos_hi = min(max(p.global_idx[(size_t)w.b * p.g + w.u0[0] + w.nvalid[0] - 1], 0), p.n - 1);
          pos_hi = max(pos_hi, pos_lo);
        }
        qblk_hi = pos_hi / p.side_block;
        qblk_lo = pos_lo / p.side_block;
        const int bias_len = p.S + (qblk_hi - qblk_lo);
        bias_staged = bias_len + 4 <= side_stride;
        if (bias_staged) {
          named_barrier_sync(3, kSoftmaxThreads);     // both groups are done with the old segment
          const float* src = p.bias + (size_t)w.h * (p.S + p.nblk - 1) + (p.nblk - 1 - qblk_hi);
          // each thread reads its values once and writes them into all four copies;
          // eight loads are in flight per thread
          const int len = (bias_len + 7) & ~3;
          for (int i0 = tid; i0 < len; i0 += 8 * kSoftmaxThreads) {
            float v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const int idx = i0 + q * kSoftmaxThreads;
              v[q] = idx < bias_len ? __ldg(src + idx) * kLog2e : 0.f;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const int idx = i0 + q * kSoftmaxThreads;
              if (idx < len) {
#pragma unroll
                for (int t = 0; t < 4; ++t)
                  if (idx - t >= 0) sSide[t * side_stride + idx - t] = v[q];
              }
            }
          }
          if (!has_local) named_barrier_sync(3, kSoftmaxThreads);
        }
      }
      if (has_local) {
        if (!bias_staged) named_barrier_sync(3, kSoftmaxThreads);   // old rows are no longer read
        const int R = p.local_radius;
        const float* tab = p.local_bias + (size_t)w.h * (2 * R + 1) + R;
        const int len = min((2 * r_eff + 2 * kLocalPad + 8) & ~3, lstride);
        for (int idx = tid; idx < len; idx += kSoftmaxThreads) {
          const int t = idx - r_eff - kLocalPad;
          const long long off = (long long)w.d * t;
          const bool in = t >= -w.r && t <= w.r && off >= -R && off <= R;
          const float val = in ? __ldg(tab + off) * kLog2e : 0.f;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            if (idx - c >= 0) sLocal[c * lstride + idx - c] = val;
        }
        named_barrier_sync(3, kSoftmaxThreads);
      }
      if (!tr.active) {
        if (MODE == 0) write_zero_row<D>(p, w, tr, row);
        continue;
      }

      const int rd = w.r * w.d;
      // random key blocks of this query tile (MODE 0, dilation 1), kept in registers
      constexpr bool has_rand = RAND && MODE == 0;
      constexpr int kRandRegs = has_rand ? kMaxRand : 1;
      int rbl[kRandRegs];
#pragma unroll
      for (int t = 0; t < kRandRegs; ++t)
        rbl[t] = (has_rand && t < p.num_rand) ? rand_block(p, w.b, tr.head, tr.u0, t) : -1;
      // this thread's position of the unit's first global-column tile, loaded early
      const int gpos0 = (GLOB && w.ngc > 0 && row < p.g) ? __ldg(p.global_idx + (size_t)w.b * p.g + row) : -1;
      int klo, khi;                            // band keys [klo, khi) of this row
      if (MODE == 0) {
        klo = u - w.r;
        khi = min(p.causal ? u : u + w.r, w.Vc - 1) + 1;
      } else {
        klo = 0;
        khi = w.key_end;
      }
      if (!row_valid) khi = klo;               // padded row: attends nothing
      const int qblk = (p.S > 0) ? pos / p.side_block : 0;
      // offset of this row's bias segment inside the staged one; it lies in range
      // whenever global_idx is sorted (clamped so that unsorted input stays in bounds)
      const int boff = min(max(qblk_hi - qblk, 0), qblk_hi - qblk_lo);
      const float* bias_row =
          has_bias ? p.bias + (size_t)w.h * (p.S + p.nblk - 1) + (p.nblk - 1 - qblk) : nullptr;

      float m = -INFINITY;                     // running max, log2 units
      float l = 0.f;
      int iu = 0;                              // tiles of this unit handled
      for (int j = 0; j < T; ++j) {
        if (!uses(w, tr, x, j)) continue;
        if (!mbar_wait_bounded(&s_full[x], it & 1, abort_v, kWaitLimitNs)) { ok = false; break; }
        tc_fence_after();
        uint32_t xr[kTile];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
          tmem_ld32(s_addr + ch * 32, *reinterpret_cast<uint32_t(*)[32]>(xr + ch * 32));
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) tmem_wait_ld_dep(*reinterpret_cast<uint32_t(*)[32]>(xr + ch * 32));
        if (C::kSepP) {
          tc_fence_before();
          mbar_arrive(&s_free[x]);             // the MMA warp may compute the next S now
        }
        float s[kTile];
#pragma unroll
        for (int e = 0; e < kTile; ++e) s[e] = __uint_as_float(xr[e]);

        // Scores: band tiles keep raw q.k (the scale is folded into the exponent);
        // global and side tiles are taken to log2 units here (plus bias * log2 e).
        // Masked entries become -inf.
        float tmax;
        bool raw = false;
        uint32_t live = 0xFu;                  // 32-column chunks with any allowed key in the warp
        if (j < w.nband) {
          const int kv0 = w.band_lo + j * kTile;
          const int lo_t = klo - kv0, hi_t = khi - kv0;
          if (has_local) {
            // s * scale + bias, in log2 units (entries outside the window are masked below)
            const int b0 = kv0 - u + r_eff + kLocalPad;
            const float* cp = sLocal + (b0 & 3) * lstride + (b0 & ~3);
#pragma unroll
            for (int e = 0; e < kTile; e += 4) {
              const float4 bb = *reinterpret_cast<const float4*>(cp + e);
              ffma2(s[e], s[e + 1], s[e], s[e + 1], sl2, sl2, bb.x, bb.y);
              ffma2(s[e + 2], s[e + 3], s[e + 2], s[e + 3], sl2, sl2, bb.z, bb.w);
            }
          }
          live = 0;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch)
            if (__any_sync(0xffffffffu, lo_t < 32 * ch + 32 && hi_t > 32 * ch)) live |= 1u << ch;
          // boundary tiles: most cut only one side of the band (window start or
          // causal diagonal), which costs one compare and one select per score
          const bool cut_lo = __any_sync(0xffffffffu, lo_t > 0);
          const bool cut_hi = __any_sync(0xffffffffu, hi_t < kTile);
          if (cut_lo && cut_hi) {
#pragma unroll
            for (int e = 0; e < kTile; ++e) s[e] = (e >= lo_t && e < hi_t) ? s[e] : -INFINITY;
          } else if (cut_lo) {
#pragma unroll
            for (int e = 0; e < kTile; ++e) s[e] = (e >= lo_t) ? s[e] : -INFINITY;
          } else if (cut_hi) {
#pragma unroll
            for (int e = 0; e < kTile; ++e) s[e] = (e < hi_t) ? s[e] : -INFINITY;
          }
          if (has_local) {
            if (!kMaxAfter) tmax = row_max128(s);
          } else {
            if (!kMaxAfter) tmax = row_max128(s) * sl2;
            raw = true;
          }
        } else if (GLOB && j < w.nband + w.ngc) {
          // global-column tile: stage its 128 positions in shared memory (one per
          // thread of the group), each with the per-key facts every row shares:
          // -1 for no key (or a key a random block of this tile already counts),
          // bit 30 set for a key of another residue class (never inside a window of
          // this tile's rows, whose positions are all c mod d).  Rows then mask the
          // keys already inside their window.
          const int e0 = (j - w.nband) * kTile;
          int code = (j == w.nband) ? gpos0
                     : ((e0 + row < p.g) ? __ldg(p.global_idx + (size_t)w.b * p.g + e0 + row) : -1);
          if (code >= 0) {
            bool in_rand = false;
            if (has_rand) {
#pragma unroll
              for (int t = 0; t < kRandRegs; ++t) in_rand = in_rand || (rbl[t] >= 0 && (code >> 7) == rbl[t]);
            }
            if (in_rand) code = -1;
            else if (w.d > 1 && code % w.d != w.c) code |= 1 << 30;
          }
          // Without the causal cut (global tokens never come with it), a key is masked iff it
          // lies beyond the g global slots or inside the row's window, |pos - key| <= rd:
          // one unsigned compare, (unsigned)(pos + rd - key) <= 2 rd.  A key of another
          // residue class is staged as a position no window reaches.  A key that a random
          // block of this tile already counts (dilation 1 there) is staged as the position
          // of the tile's middle row, which every row's window holds when r >= 64.
          const bool fast = !p.causal && (!has_rand || w.r >= kTile / 2);
          if (fast) {
            if (code >= 0) code = (code & (1 << 30)) ? -(1 << 29) : code;
            else if (has_rand) code = w.c + w.d * (tr.u0 + kTile / 2);
          }
          named_barrier_sync(1 + x, 128);      // the previous tile's readers are done
          sGpos[x * kTile + row] = code;
          named_barrier_sync(1 + x, 128);
          if (fast) {
            const int posr = pos + rd;
            const unsigned span = 2u * (unsigned)rd;
            const int glim = row_valid ? p.g - e0 : 0;     // slots of this tile that hold a key
#pragma unroll
            for (int e = 0; e < kTile; e += 4) {
              const int4 kp = *reinterpret_cast<const int4*>(&sGpos[x * kTile + e]);
              s[e] = (e < glim && (unsigned)(posr - kp.x) > span) ? s[e] * sl2 : -INFINITY;
              s[e + 1] = (e + 1 < glim && (unsigned)(posr - kp.y) > span) ? s[e + 1] * sl2 : -INFINITY;
              s[e + 2] = (e + 2 < glim && (unsigned)(posr - kp.z) > span) ? s[e + 2] * sl2 : -INFINITY;
              s[e + 3] = (e + 3 < glim && (unsigned)(posr - kp.w) > span) ? s[e + 3] * sl2 : -INFINITY;
            }
          } else {
#pragma unroll
            for (int e = 0; e < kTile; ++e) {
              const int cv = sGpos[x * kTile + e];
              const int diff = pos - (cv & ~(1 << 30));
              const bool inwin =
                  !(cv & (1 << 30)) && (p.causal ? (diff >= 0 && diff <= rd) : (abs(diff) <= rd));
              const bool allowed = row_valid && cv >= 0 && !inwin;
              s[e] = allowed ? s[e] * sl2 : -INFINITY;
            }
          }
          if (!kMaxAfter) tmax = row_max128(s);
        } else if (has_rand && j >= w.rand0) {
          // random key block: keys below the valid length and outside the row's
          // window; a block repeated earlier in the list is masked whole
          int t;
          rand_owner(w, j, t);
          int kb = -1;
#pragma unroll
          for (int t2 = 0; t2 < kRandRegs; ++t2)
            if (t2 == t) kb = rbl[t2];
          // an index outside the key blocks attends nothing (masked like a repeat)
          bool dup = kb < 0 || kb * kTile >= p.n;
#pragma unroll
          for (int t2 = 0; t2 < kRandRegs; ++t2) dup = dup || (t2 < t && rbl[t2] == kb);
          const int kv0 = kb * kTile;
          const int lo_t = klo - kv0, hi_t = khi - kv0, v_t = w.Vc - kv0;
          // key e counts iff e < vlim (the valid keys of a live row and block) and it lies
          // outside the row's window [lo_t, hi_t): (unsigned)(e - lo_t) >= hi_t - lo_t
          const int vlim = (row_valid && !dup) ? v_t : 0;
          const unsigned span = (unsigned)max(hi_t - lo_t, 0);
#pragma unroll
          for (int e = 0; e < kTile; ++e)
            s[e] = (e < vlim && (unsigned)(e - lo_t) >= span) ? s[e] * sl2 : -INFINITY;
          live = 0;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch)
            if (__any_sync(0xffffffffu, row_valid && !dup && 32 * ch < v_t)) live |= 1u << ch;
          if (!kMaxAfter) tmax = row_max128(s);
        } else {
          const int s0 = (j - w.nband - w.ngc) * kTile;
          const int lim = row_valid ? p.S - s0 : 0;
          if (bias_row && bias_staged) {
            const int b0 = s0 + boff;
            const float* cp = sSide + (b0 & 3) * side_stride + (b0 & ~3);
#pragma unroll
            for (int e = 0; e < kTile; e += 4) {
              const float4 bb = *reinterpret_cast<const float4*>(cp + e);
              ffma2(s[e], s[e + 1], s[e], s[e + 1], sl2, sl2, bb.x, bb.y);
              ffma2(s[e + 2], s[e + 3], s[e + 2], s[e + 3], sl2, sl2, bb.z, bb.w);
            }
          } else if (bias_row) {
            // segment too long to stage: read the bias from global memory, 16 at a time
#pragma unroll
            for (int e = 0; e < kTile; e += 16) {
#pragma unroll
              for (int q = 0; q < 16; ++q)
                s[e + q] = s[e + q] * sl2 + (e + q < lim ? __ldg(bias_row + s0 + e + q) : 0.f) * kLog2e;
              asm volatile("" ::: "memory");
            }
          } else {
#pragma unroll
            for (int e = 0; e < kTile; e += 2) ffma2(s[e], s[e + 1], s[e], s[e + 1], sl2, sl2, 0.f, 0.f);
          }
          if (!__all_sync(0xffffffffu, lim >= kTile)) {
#pragma unroll
            for (int e = 0; e < kTile; ++e) s[e] = e < lim ? s[e] : -INFINITY;
            live = 0;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch)
              if (__any_sync(0xffffffffu, 32 * ch < lim)) live |= 1u << ch;
          }
          if (!kMaxAfter) tmax = row_max128(s);
        }

        // Online softmax with a lazy rescale: the reference max m only moves when
        // the tile max exceeds it by more than 2^8 (l and O always share m).
        if (kMaxAfter) tmax = row_max128(s) * (raw ? sl2 : 1.f);
        const float m_new = fmaxf(m, tmax);
        const bool need = (m == -INFINITY) ? (m_new > -INFINITY) : (m_new > m + kRescaleThreshold);
        const bool rescale = __any_sync(0xffffffffu, need);
        float alpha = 1.f;
        if (rescale) {
          alpha = (m == -INFINITY) ? 0.f : ex2_approx(m - m_new);
          l *= alpha;
          m = m_new;
        }
        const float neg_m = (m == -INFINITY) ? 0.f : -m;
        const float mul = raw ? sl2 : 1.f;
        if (C::kSepP && pw > 0) {
          // the previous PV has read P_x and updated O_x
          if (!mbar_wait_bounded(&pv_done[x], (pw - 1) & 1, abort_v, kWaitLimitNs)) { ok = false; break; }
          tc_fence_after();
        }
        if (!C::kSepP && rescale && iu > 0) {
          // P over S: O_x must be rescaled before the first half of P is published.
          // It is stable: its previous PV was issued before this S and MMAs complete
          // in order.  (16 columns at a time: the scores are still live in registers.)
#pragma unroll 1
          for (int ch = 0; ch < D / 16; ++ch) {
            uint32_t rr[16];
            tmem_ld16(o_addr + ch * 16, rr);
            tmem_wait_ld_dep16(rr);
#pragma unroll
            for (int e = 0; e < 16; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * alpha);
            tmem_st16(o_addr + ch * 16, rr);
          }
        }
        float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
        // P = 2^(t - m) as bf16, written 16 columns at a time (over S: the columns of
        // chunk c only hold S values already read into registers)
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t pk[16];
          if (!(live & (1u << ch))) {
            // every key of this chunk is masked for every row of the warp: P = 0
#pragma unroll
            for (int q = 0; q < 16; ++q) pk[q] = 0u;
          } else {
#pragma unroll
            for (int q = 0; q < 32; q += 4) {
              const int e = ch * 32 + q;
              float a0, a1, a2, a3;
              ffma2(a0, a1, s[e], s[e + 1], mul, mul, neg_m, neg_m);
              ffma2(a2, a3, s[e + 2], s[e + 3], mul, mul, neg_m, neg_m);
              if (q < emu_per32<D>()) {
                exp2_poly2(a0, a1, a0, a1);
                exp2_poly2(a2, a3, a2, a3);
              } else {
                a0 = ex2_approx(a0);
                a1 = ex2_approx(a1);
                a2 = ex2_approx(a2);
                a3 = ex2_approx(a3);
              }
              fadd2(acc0, acc1, acc0, acc1, a0, a1);
              fadd2(acc2, acc3, acc2, acc3, a2, a3);
              pk[q / 2] = pack_bf16x2(a0, a1);
              pk[q / 2 + 1] = pack_bf16x2(a2, a3);
            }
          }
          tmem_st16(p_addr + ch * 16, pk);
          if (!C::kSepP && ch == 1) {
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&p_half[x]);
          }
        }
        l += (acc0 + acc1) + (acc2 + acc3);
        if (C::kSepP && rescale && iu > 0) {
          // separate P: the wait on the previous PV above saw O_x updated
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t rr[32];
            tmem_ld32(o_addr + ch * 32, rr);
            tmem_wait_ld_dep(rr);
#pragma unroll
            for (int e = 0; e < 32; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * alpha);
            tmem_st32(o_addr + ch * 32, rr);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[x]);
        ++pw;
        ++it;
        ++iu;
      }
      if (!ok) break;

      // ---------------------------------------------------------- epilogue
      // O_x is read out of TMEM before this group's next p_full arrival, which is
      // what the MMA warp waits for before it overwrites O_x.
      if (!mbar_wait_bounded(&o_full[x], oc & 1, abort_v, kWaitLimitNs)) { ok = false; break; }
      ++oc;
      tc_fence_after();
      const bool has = row_valid && l > 0.f;
      const float inv = has ? 1.f / l : 0.f;
      const float lse_v = has ? (m + __log2f(l)) * kLn2 : -INFINITY;
      if (MODE == 0 && !has_bias && !has_local) {
        // Coalesced store: 32-column chunks staged in shared memory (the bias area,
        // unused without biases; two 8 KB buffers per group, 64-byte swizzle)
        // and written by TMA; rows beyond the class end are clipped by the map.
        uint8_t* stage = reinterpret_cast<uint8_t*>(sBias) + x * 2 * 8192;
        if (row == 0) tma_store_wait_read<0>();          // previous unit's stores have read
        named_barrier_sync(1 + x, 128);
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint8_t* buf = stage + (ch & 1) * 8192;
          if (ch >= 2) {
            if (row == 0) tma_store_wait_read<1>();      // the store of chunk ch-2 has read buf
            named_barrier_sync(1 + x, 128);
          }
          uint32_t rr[32];
          tmem_ld32(o_addr + ch * 32, rr);
          tmem_wait_ld_dep(rr);
          uint8_t* rbase = buf + row * 64;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 0]) * inv, __uint_as_float(rr[q4 * 8 + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 2]) * inv, __uint_as_float(rr[q4 * 8 + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 4]) * inv, __uint_as_float(rr[q4 * 8 + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 6]) * inv, __uint_as_float(rr[q4 * 8 + 7]) * inv);
            *reinterpret_cast<uint4*>(rbase + ((q4 ^ ((row >> 1) & 3)) << 4)) = v;
          }
          fence_proxy_async_smem();
          named_barrier_sync(1 + x, 128);
          if (row == 0) {
            tma_store_3d(&p.mo[w.cls], buf, ch * 32, tr.u0, w.b * p.Hq + tr.head);
            tma_store_commit();
          }
        }
        if (row < tr.rows && p.lse) p.lse[out_row(p, w, tr, row)] = lse_v;
      } else if (MODE == 0) {
        const size_t off = out_row(p, w, tr, row);
        uint4* orow = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + off * D);
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t rr[32];
          tmem_ld32(o_addr + ch * 32, rr);
          tmem_wait_ld_dep(rr);
          if (row < tr.rows) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 0]) * inv, __uint_as_float(rr[q4 * 8 + 1]) * inv);
              v.y = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 2]) * inv, __uint_as_float(rr[q4 * 8 + 3]) * inv);
              v.z = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 4]) * inv, __uint_as_float(rr[q4 * 8 + 5]) * inv);
              v.w = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 6]) * inv, __uint_as_float(rr[q4 * 8 + 7]) * inv);
              orow[ch * 4 + q4] = v;
            }
          }
        }
        if (row < tr.rows && p.lse) p.lse[off] = lse_v;
      } else {
        const size_t prow =
            ((size_t)w.split * p.B * p.Hq + (size_t)w.b * p.Hq + w.h) * p.gpad + w.u0[0] + row;
        float4* po = reinterpret_cast<float4*>(p.part_o + prow * D);
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t rr[32];
          tmem_ld32(o_addr + ch * 32, rr);
          tmem_wait_ld_dep(rr);
          if (row < w.rows[0]) {
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              po[ch * 8 + q4] = make_float4(__uint_as_float(rr[q4 * 4 + 0]) * inv, __uint_as_float(rr[q4 * 4 + 1]) * inv,
                                            __uint_as_float(rr[q4 * 4 + 2]) * inv, __uint_as_float(rr[q4 * 4 + 3]) * inv);
          }
        }
        if (row < w.rows[0]) p.part_lse[prow] = lse_v;
      }
      tc_fence_before();
    }
  }

  if (warp < 8 && (tid & 127) == 0) tma_store_wait_read<0>();   // staged stores have read smem
  if (MODE == 1) grid_dependency_wait();    // the band grid, before the merge behind this one
  tc_fence_before();
  __syncthreads();
  if (abort_flag) {
    // A bounded wait expired: report it, then give copies and MMAs still in
    // flight time to land before TMEM and shared memory are released.
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


}  // namespace

size_t band_tc_smem_bytes(int D) {
  return D == 64 ? Cfg<64>::kSmemBytes : Cfg<128>::kSmemBytes;
}

template <int D, int MODE, bool LOCAL = false, bool RAND = false, bool AGG = false, bool GLOB = true>
static cudaError_t launch_one(const AttnParams& p, int units, int num_sms, cudaStream_t s, bool pdl = false) {
  auto kern = attn_tc_kernel<D, MODE, LOCAL, RAND, AGG, GLOB>;
  const int smem = static_cast<int>(Cfg<D>::kSmemBytes);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int grid = units < num_sms ? units : num_sms;
  if (grid <= 0) return cudaSuccess;
  if (AGG) {
    // the prologue's wait needs every CTA resident at once: a cooperative launch
    // (one CTA per SM, grid <= SM count)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
  }
  if (pdl) {
    // programmatic dependent launch: scheduled while the previous kernel drains
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
  }
  kern<<<grid, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

// p.tiles[h] holds the number of two-tile units of head h, p.max_units their maximum.
// The band kernel for one value of GLOB (global-column tiles present or not).
template <bool GLOB>
static cudaError_t launch_band_variant(const AttnParams& p, int units, int num_sms, cudaStream_t s) {
  if (p.agg_count) {      // side keys built in the prologue (no local bias, no random blocks)
    return p.D == 64 ? launch_one<64, 0, false, false, true, GLOB>(p, units, num_sms, s)
                     : launch_one<128, 0, false, false, true, GLOB>(p, units, num_sms, s);
  }
  if (p.num_rand > 0) {
    if (p.local_bias)
      return p.D == 64 ? launch_one<64, 0, true, true, false, GLOB>(p, units, num_sms, s, GLOB)
                       : launch_one<128, 0, true, true, false, GLOB>(p, units, num_sms, s, GLOB);
    return p.D == 64 ? launch_one<64, 0, false, true, false, GLOB>(p, units, num_sms, s, GLOB)
                     : launch_one<128, 0, false, true, false, GLOB>(p, units, num_sms, s, GLOB);
  }
  if (p.local_bias)
    return p.D == 64 ? launch_one<64, 0, true, false, false, GLOB>(p, units, num_sms, s, GLOB)
                     : launch_one<128, 0, true, false, false, GLOB>(p, units, num_sms, s, GLOB);
  return p.D == 64 ? launch_one<64, 0, false, false, false, GLOB>(p, units, num_sms, s, GLOB)
                   : launch_one<128, 0, false, false, false, GLOB>(p, units, num_sms, s, GLOB);
}

cudaError_t launch_band_tc(const AttnParams& p, int num_sms, cudaStream_t s) {
  const int units = p.max_units * p.B * p.Hq;
  return p.g > 0 ? launch_band_variant<true>(p, units, num_sms, s)
                 : launch_band_variant<false>(p, units, num_sms, s);
}

cudaError_t launch_global_rows_tc(const AttnParams& p, int num_sms, cudaStream_t s) {
  const int units = p.nsplit * (p.gpad / kTile) * p.B * p.Hq;
  return p.D == 64 ? launch_one<64, 1>(p, units, num_sms, s, true) : launch_one<128, 1>(p, units, num_sms, s, true);
}

int band_bias_copy(int) { return kBiasCopy; }

}  // namespace swa
