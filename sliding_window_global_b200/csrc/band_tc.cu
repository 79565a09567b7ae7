// band_tc.cu -- tcgen05 (5th-generation tensor core) kernel for banded sparse
// self-attention on sm_100a: bf16 inputs, fp32 accumulation in TMEM.
//
// One CTA owns a unit of two 128-row query tiles (A and B, consecutive rows) of
// one (batch, query head, residue class) and walks a list of 128-key tiles:
//   band tiles   -- keys of the (dilated, optionally causal) sliding window
//                   ("精读笔记：Big Bird" §3.2.1; the Longformer page §二 for
//                   dilation; SWAN-GPT §3.3(1) for the causal 512-key window); only
//                   the tiles the two windows touch are loaded, so fully masked
//                   tiles are skipped and each K/V tile feeds both query tiles;
//   global tiles -- the gathered global tokens every query also attends to,
//                   minus those already inside its window (BigBird §3.2.3, ITC);
//   side tiles   -- appended side keys with the additive bucketed bias of the
//                   LongT5 Transient-Global attention ("LongT5 长序列模型完全指南",
//                   Transient-Global and 源码级证据 sections).
// With dilation d a query at position c + d*u only meets keys c + d*u', so each
// residue class is a plain band of radius r over rows c, c+d, ..., read and
// written through strided TMA tensor maps.
//
// MODE 1 computes global query rows (full attention over all valid keys, plus
// side keys), split over key ranges into fp32 partials that a logsumexp merge
// combines; there tile B is unused.
//
// Warp roles (320 threads):
//   warps 0-3   softmax of tile A, warps 4-7 softmax of tile B: thread t of the
//               group owns query row t (TMEM lane t).  Per key tile: load S from
//               TMEM, mask (boundary tiles only), scale, add bias (side tiles),
//               running max m / sum l with a lazy O rescale (only when the max
//               grows by more than 2^8), exponentiate, write P (bf16) back into
//               the TMEM columns of S.  At the end: O / l -> bf16 -> TMA store.
//   warp 8      TMA producer: Q_A, Q_B once, then K/V tiles into an NS-stage ring.
//   warp 9      TMEM allocator and MMA issuer.  Per key tile j it issues, for A
//               then B: O += P(j) V(j) (A operand P read from TMEM), immediately
//               followed by S = Q K(j+1)^T into the same TMEM columns, so the
//               tensor core works on one query tile while the other one's softmax
//               runs (ping-pong).  MMAs issued by one thread execute in order, so
//               the next S never overwrites a P that an earlier MMA still reads.
#include "ptx.cuh"
#include "swa_kernels.h"

namespace swa {
namespace {

constexpr int kSoftmaxThreads = 256;
constexpr int kThreads = 320;
constexpr uint32_t kSub = 128 * 128;          // one 128-row x 128-byte swizzle sub-tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;     // log2 units
constexpr int kBiasCopy = 2048;               // floats per shifted copy of the side-bias segment

template <int D>
struct Cfg {
  static constexpr int NS = (D == 64) ? 4 : 2;                 // K/V ring stages
  static constexpr uint32_t kTileBytes = 128u * D * 2u;        // one 128 x D bf16 tile
  static constexpr uint32_t kQOff = 0;                         // Q_A, Q_B (reused for O staging)
  static constexpr uint32_t kKOff = 2 * kTileBytes;
  static constexpr uint32_t kVOff = kKOff + NS * kTileBytes;
  static constexpr uint32_t kBiasOff = kVOff + NS * kTileBytes;  // 4 shifted copies
  static constexpr uint32_t kBarOff = kBiasOff + 4 * kBiasCopy * 4;
  static constexpr int kNumBars = 1 + 3 * NS + 6;
  static constexpr uint32_t kSmemBytes = kBarOff + kNumBars * 8 + 1024;
  static constexpr uint32_t kTmemCols = 512;                    // S_A | S_B | O_A | O_B
  __host__ __device__ static constexpr uint32_t s_col(int x) { return x ? 128u : 0u; }
  __host__ __device__ static constexpr uint32_t o_col(int x) { return 256u + (x ? D : 0); }
};

// ------------------------------------------------------------------ work description
struct Work {
  int b, h, hk, cls, d, c, r;
  int u0[2];            // first row (class coordinates / global slot) of tile A, B
  int rows[2];          // rows that exist
  int valid[2];         // rows below the valid length / below g
  int Vc;               // valid rows of the class (MODE 0) / valid keys (MODE 1)
  int split;            // MODE 1 key split
  bool active[2];
  int band_lo;          // first key of band tile 0
  int nband, ngc, nside, total;
  int key_end;          // MODE 1: keys at or beyond this are masked
  int lo[2], hi[2];     // band key range of each query tile (class coordinates)
};

template <int MODE>
__device__ __forceinline__ bool decode_work(const AttnParams& p, Work& w) {
  if (MODE == 0) {
    w.b = blockIdx.z;
    w.h = blockIdx.y;
    int unit = blockIdx.x;
    if (unit >= p.tiles[w.h]) return false;    // p.tiles holds two-tile units per head
    w.hk = w.h / p.G;
    w.r = p.window[w.h];
    const int base = p.class_base[w.h];
    w.d = p.cls[base].d;
    int c = 0;
    for (; c < w.d; ++c) {
      const int tc = (p.cls[base + c].n_c + kTile - 1) / kTile;
      const int uc = (tc + 1) / 2;
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
      w.u0[x] = unit * 2 * kTile + x * kTile;
      w.rows[x] = max(0, min(kTile, nc - w.u0[x]));
      w.valid[x] = max(0, min(w.rows[x], w.Vc - w.u0[x]));
      w.active[x] = w.valid[x] > 0;
      w.lo[x] = max(0, w.u0[x] - w.r);
      const int last = w.u0[x] + w.valid[x] - 1;
      w.hi[x] = p.causal ? min(w.Vc, last + 1) : min(w.Vc, last + w.r + 1);
    }
    w.band_lo = w.lo[0];
    const int hi = w.active[1] ? max(w.hi[0], w.hi[1]) : w.hi[0];
    w.nband = w.active[0] ? (hi - w.band_lo + kTile - 1) / kTile : 0;
    w.ngc = (w.active[0] && p.g > 0) ? (p.g + kTile - 1) / kTile : 0;
    w.nside = (w.active[0] && p.S > 0) ? (p.S + kTile - 1) / kTile : 0;
  } else {
    w.split = blockIdx.x;
    const int gt = blockIdx.y;
    const int bh = blockIdx.z;
    w.b = bh / p.Hq;
    w.h = bh % p.Hq;
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
    w.valid[0] = max(0, min(w.rows[0], p.g - w.u0[0]));
    w.u0[1] = 0;
    w.rows[1] = w.valid[1] = 0;
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
    w.active[0] = w.valid[0] > 0 && (w.nband + w.nside) > 0;
    if (!w.active[0]) w.nband = w.nside = 0;
    w.lo[0] = w.band_lo;
    w.hi[0] = w.key_end;
    w.lo[1] = w.hi[1] = 0;
  }
  w.total = w.nband + w.ngc + w.nside;
  return true;
}

// Does query tile x use key tile j?
__device__ __forceinline__ bool uses(const Work& w, int x, int j) {
  if (!w.active[x] || j >= w.total) return false;
  if (j >= w.nband) return true;                        // global and side tiles: every row
  const int kv0 = w.band_lo + j * kTile;
  return kv0 < w.hi[x] && kv0 + kTile > w.lo[x];
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
  } else {
    mk = &p.msk;
    mv = &p.msv;
    y = (j - w.nband - w.ngc) * kTile;
  }
}

template <int D>
__device__ __forceinline__ void tma_tile(void* dst, const CUtensorMap* map, uint64_t* bar, int y,
                                         int z) {
  tma_load_3d(dst, map, bar, 0, y, z);
  if (D == 128) tma_load_3d(static_cast<uint8_t*>(dst) + kSub, map, bar, 64, y, z);
}

template <int D>
__device__ __forceinline__ void tma_store_tile(const CUtensorMap* map, const void* src, int y, int z) {
  tma_store_3d(map, src, 0, y, z);
  if (D == 128) tma_store_3d(map, static_cast<const uint8_t*>(src) + kSub, 64, y, z);
}

// ------------------------------------------------------------------ packed fp32 helpers
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1,
                                      float c0, float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void fadd2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
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

// ------------------------------------------------------------------ padding rows
template <int D>
__device__ void write_zero_row(const AttnParams& p, const Work& w, int x, int row) {
  if (row >= w.rows[x] || row < w.valid[x]) return;
  const int pos = w.c + w.d * (w.u0[x] + row);
  const size_t off = ((size_t)(w.b * p.Hq + w.h) * p.n + pos);
  uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + off * D);
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i] = make_uint4(0, 0, 0, 0);
  if (p.lse) p.lse[off] = -INFINITY;
}

template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ AttnParams p) {
  using C = Cfg<D>;
  constexpr int NS = C::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + C::kQOff;
  uint8_t* sK = smem + C::kKOff;
  uint8_t* sV = smem + C::kVOff;
  float* sBias = reinterpret_cast<float*>(smem + C::kBiasOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + NS;
  uint64_t* kv_empty = v_full + NS;
  uint64_t* s_full = kv_empty + NS;       // [2]
  uint64_t* p_full = s_full + 2;          // [2]
  uint64_t* o_full = p_full + 2;          // [2]
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int sGpos[2 * kTile];          // global positions of the current global tile

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  Work w;
  if (!decode_work<MODE>(p, w)) return;

  if (!w.active[0]) {
    if (MODE == 0) {
      if (tid < kSoftmaxThreads) write_zero_row<D>(p, w, tid >> 7, tid & 127);
    } else if (tid < kTile) {
      const int slot = w.u0[0] + tid;
      if (slot < p.gpad) {
        const size_t prow = ((size_t)w.split * p.B * p.Hq + (size_t)w.b * p.Hq + w.h) * p.gpad + slot;
        float4* po = reinterpret_cast<float4*>(p.part_o + prow * D);
        for (int i = 0; i < D / 4; ++i) po[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        p.part_lse[prow] = -INFINITY;
      }
    }
    return;
  }

  const int T = w.total;

  // side-bias staging parameters (CTA-uniform)
  int qblk_hi = 0, bias_len = 0;
  bool bias_staged = false;
  if (p.bias && p.S > 0) {
    int pos_lo, pos_hi;
    if (MODE == 0) {
      const int last_row = w.active[1] ? w.u0[1] + w.valid[1] - 1 : w.u0[0] + w.valid[0] - 1;
      pos_lo = w.c + w.d * w.u0[0];
      pos_hi = w.c + w.d * last_row;
    } else {
      pos_lo = p.global_idx[(size_t)w.b * p.g + w.u0[0]];
      pos_hi = p.global_idx[(size_t)w.b * p.g + w.u0[0] + w.valid[0] - 1];
    }
    const int qblk_lo = pos_lo / p.side_block;
    qblk_hi = pos_hi / p.side_block;
    bias_len = p.S + (qblk_hi - qblk_lo);
    bias_staged = bias_len + 4 <= kBiasCopy;
  }

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], kTile);
      mbar_init(&o_full[x], 1);
    }
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(&tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  if (bias_staged && tid < kSoftmaxThreads) {
    // copy t holds seg[x + t]; seg[i] = log2(e) * bias[h][i + nblk - 1 - qblk_hi]
    const float* src = p.bias + (size_t)w.h * (p.S + p.nblk - 1) + (p.nblk - 1 - qblk_hi);
    for (int i = tid; i < 4 * kBiasCopy; i += kSoftmaxThreads) {
      const int t = i / kBiasCopy, xx = i % kBiasCopy;
      const int idx = xx + t;
      sBias[i] = idx < bias_len ? __ldg(src + idx) * kLog2e : 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int* abort_v = &abort_flag;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const CUtensorMap* mq = (MODE == 0) ? &p.mq[w.cls] : &p.mgq;
      const int qz = w.b * p.Hq + w.h;
      const int kz = w.b * p.Hkv + w.hk;
      mbar_arrive_expect_tx(q_full, (w.active[1] ? 2u : 1u) * C::kTileBytes);
      tma_tile<D>(sQ, mq, q_full, w.u0[0], qz);
      if (w.active[1]) tma_tile<D>(sQ + C::kTileBytes, mq, q_full, w.u0[1], qz);
      for (int j = 0; j < T; ++j) {
        const int st = j % NS;
        const int use = j / NS;
        if (j >= NS && !mbar_wait_bounded(&kv_empty[st], (use - 1) & 1, abort_v, kWaitLimitNs)) break;
        const CUtensorMap *mk, *mv;
        int y;
        tile_source(p, w, j, mk, mv, y);
        mbar_arrive_expect_tx(&k_full[st], C::kTileBytes);
        tma_tile<D>(sK + st * C::kTileBytes, mk, &k_full[st], y, kz);
        mbar_arrive_expect_tx(&v_full[st], C::kTileBytes);
        tma_tile<D>(sV + st * C::kTileBytes, mv, &v_full[st], y, kz);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t k_base = smem_u32(sK);
      const uint32_t v_base = smem_u32(sV);
      int issued[2] = {-1, -1};
      int npv[2] = {0, 0};
      int last[2] = {-1, -1};
      for (int x = 0; x < 2; ++x)
        for (int j = 0; j < T; ++j)
          if (uses(w, x, j)) last[x] = j;
      bool ok = mbar_wait_bounded(q_full, 0, abort_v, kWaitLimitNs);
      auto issue_qk = [&](int x, int j) -> bool {
        if (!mbar_wait_bounded(&k_full[j % NS], (j / NS) & 1, abort_v, kWaitLimitNs)) return false;
        tc_fence_after();
        const uint32_t qt = q_base + x * C::kTileBytes;
        const uint32_t kt = k_base + (j % NS) * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kSub + (kk & 3) * 32;
          umma_ss(tmem + C::s_col(x), sdesc_sw128(qt + off, 16, 1024), sdesc_sw128(kt + off, 16, 1024),
                  idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[x]);
        issued[x] = j;
        return true;
      };
      for (int j = 0; ok && j < T; ++j) {
        const int st = j % NS;
        for (int x = 0; x < 2 && ok; ++x)
          if (uses(w, x, j) && issued[x] < j) ok = issue_qk(x, j);
        if (!ok) break;
        if (!mbar_wait_bounded(&v_full[st], (j / NS) & 1, abort_v, kWaitLimitNs)) { ok = false; break; }
        const uint32_t vt = v_base + st * C::kTileBytes;
        for (int x = 0; x < 2 && ok; ++x) {
          if (!uses(w, x, j)) continue;
          if (!mbar_wait_bounded(&p_full[x], npv[x] & 1, abort_v, kWaitLimitNs)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            umma_ts(tmem + C::o_col(x), tmem + C::s_col(x) + kk * 8,
                    sdesc_sw128(vt + kk * 2048, kSub, 1024), idesc_pv, (npv[x] > 0 || kk > 0) ? 1u : 0u);
          ++npv[x];
          if (j == last[x]) umma_commit(&o_full[x]);
          else if (uses(w, x, j + 1)) ok = issue_qk(x, j + 1);
        }
        umma_commit(&kv_empty[st]);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int x = warp >> 2;                   // 0: tile A, 1: tile B
    const int row = tid & 127;                 // TMEM lane == row in the tile
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t s_addr = lane_base + C::s_col(x);
    const uint32_t o_addr = lane_base + C::o_col(x);
    const bool tile_on = w.active[x];
    const bool row_valid = row < w.valid[x];
    const int u = w.u0[x] + row;
    int pos = 0;
    if (MODE == 0) pos = w.c + w.d * u;
    else if (row_valid) pos = p.global_idx[(size_t)w.b * p.g + w.u0[0] + row];
    const int rd = w.r * w.d;
    const float sl2 = p.scale_log2;
    // band mask range of this row, in key coordinates
    int klo, khi;
    if (MODE == 0) {
      klo = u - w.r;
      khi = min(p.causal ? u : u + w.r, w.Vc - 1) + 1;
    } else {
      klo = 0;
      khi = w.key_end;
    }
    if (!row_valid) khi = klo;                 // padded row: attends nothing
    // side-bias source for this row
    const int qblk = (p.S > 0) ? pos / p.side_block : 0;
    const int boff = qblk_hi - qblk;
    const float* bias_row =
        (p.bias && p.S > 0) ? p.bias + (size_t)w.h * (p.S + p.nblk - 1) + (p.nblk - 1 - qblk) : nullptr;

    float m = -INFINITY;                       // running max, log2 units
    float l = 0.f;
    int it = 0;
    bool ok = true;
    for (int j = 0; tile_on && j < T; ++j) {
      if (!uses(w, x, j)) continue;
      if (!mbar_wait_bounded(&s_full[x], it & 1, abort_v, kWaitLimitNs)) { ok = false; break; }
      tc_fence_after();
      uint32_t xr[kTile];
#pragma unroll
      for (int ch = 0; ch < 4; ++ch)
        tmem_ld32(s_addr + ch * 32, *reinterpret_cast<uint32_t(*)[32]>(xr + ch * 32));
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) tmem_wait_ld_dep(*reinterpret_cast<uint32_t(*)[32]>(xr + ch * 32));
      float s[kTile];
#pragma unroll
      for (int e = 0; e < kTile; ++e) s[e] = __uint_as_float(xr[e]);

      // Scores: band tiles keep raw q.k (the scale is folded into the exponent);
      // global and side tiles are taken to log2 units here (plus bias * log2 e).
      // Masked entries become -inf.
      float tmax;
      bool raw = false;
      if (j < w.nband) {
        const int kv0 = w.band_lo + j * kTile;
        const int lo_t = klo - kv0, hi_t = khi - kv0;
        const bool interior = (lo_t <= 0) && (hi_t >= kTile);
        if (!__all_sync(0xffffffffu, interior)) {
#pragma unroll
          for (int e = 0; e < kTile; ++e) s[e] = (e >= lo_t && e < hi_t) ? s[e] : -INFINITY;
        }
        tmax = row_max128(s) * sl2;
        raw = true;
      } else if (j < w.nband + w.ngc) {
        // global-column tile: stage its 128 positions in shared memory (one per
        // thread of the group), then mask the keys already inside the window
        const int e0 = (j - w.nband) * kTile;
        named_barrier_sync(1 + x, 128);        // previous tile's readers are done
        sGpos[x * kTile + row] = (e0 + row < p.g) ? __ldg(p.global_idx + (size_t)w.b * p.g + e0 + row) : -1;
        named_barrier_sync(1 + x, 128);
#pragma unroll
        for (int e = 0; e < kTile; ++e) {
          const int gp = sGpos[x * kTile + e];
          const int diff = pos - gp;
          bool inwin = p.causal ? (diff >= 0 && diff <= rd) : (abs(diff) <= rd);
          inwin = inwin && (diff % w.d == 0);
          const bool allowed = row_valid && gp >= 0 && !inwin;
          s[e] = allowed ? s[e] * sl2 : -INFINITY;
        }
        tmax = row_max128(s);
      } else {
        const int s0 = (j - w.nband - w.ngc) * kTile;
        const int lim = row_valid ? p.S - s0 : 0;
        if (bias_row && bias_staged) {
          const int b0 = s0 + boff;
          const float* cp = sBias + (b0 & 3) * kBiasCopy + (b0 & ~3);
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
        }
        tmax = row_max128(s);
      }

      // Online softmax with a lazy rescale: the reference max m only moves when the
      // tile max exceeds it by more than 2^8 (the sum l and O always share m).
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
      float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
      // P = 2^(t - m) as bf16, written back over the S columns 16 at a time (the
      // columns of chunk c only hold S values already read into registers)
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t pk[16];
#pragma unroll
        for (int q = 0; q < 32; q += 4) {
          const int e = ch * 32 + q;
          float a0, a1, a2, a3;
          ffma2(a0, a1, s[e], s[e + 1], mul, mul, neg_m, neg_m);
          ffma2(a2, a3, s[e + 2], s[e + 3], mul, mul, neg_m, neg_m);
          a0 = ex2_approx(a0);
          a1 = ex2_approx(a1);
          a2 = ex2_approx(a2);
          a3 = ex2_approx(a3);
          fadd2(acc0, acc1, acc0, acc1, a0, a1);
          fadd2(acc2, acc3, acc2, acc3, a2, a3);
          pk[q / 2] = pack_bf16x2(a0, a1);
          pk[q / 2 + 1] = pack_bf16x2(a2, a3);
        }
        tmem_st16(s_addr + ch * 16, pk);
      }
      l += (acc0 + acc1) + (acc2 + acc3);
      if (rescale && it > 0) {
        // O_x is stable: its previous PV was issued before this S, and MMAs
        // complete in order.
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
      ++it;
    }

    // ------------------------------------------------------------ epilogue
    if (tile_on) {
      const bool got = ok && mbar_wait_bounded(&o_full[x], 0, abort_v, kWaitLimitNs);
      tc_fence_after();
      const bool has = row_valid && l > 0.f;
      const float inv = has ? 1.f / l : 0.f;
      const float lse_v = has ? (m + __log2f(l)) * kLn2 : -INFINITY;
      if (MODE == 0) {
        uint8_t* stage = sQ + x * C::kTileBytes;        // Q_x is dead: every QK_x completed
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t rr[32];
          if (got) {
            tmem_ld32(o_addr + ch * 32, rr);
            tmem_wait_ld_dep(rr);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) rr[e] = 0u;
          }
          // columns ch*32 .. ch*32+31 -> 64-column sub-tile, four 16-byte chunks
          uint8_t* sub = stage + ((ch * 32) >> 6) * kSub + row * 128;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int chunk = (((ch * 32) & 63) >> 3) + q4;
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 0]) * inv, __uint_as_float(rr[q4 * 8 + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 2]) * inv, __uint_as_float(rr[q4 * 8 + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 4]) * inv, __uint_as_float(rr[q4 * 8 + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 6]) * inv, __uint_as_float(rr[q4 * 8 + 7]) * inv);
            *reinterpret_cast<uint4*>(sub + ((chunk ^ (row & 7)) << 4)) = v;
          }
        }
        if (row < w.rows[x] && p.lse) p.lse[(size_t)(w.b * p.Hq + w.h) * p.n + pos] = lse_v;
        fence_proxy_async_smem();
        named_barrier_sync(1 + x, 128);
        if (row == 0) {
          // the class map of q doubles as the map of out (same shape and strides)
          tma_store_tile<D>(&p.mo[w.cls], stage, w.u0[x], w.b * p.Hq + w.h);
          tma_store_commit_and_wait();
        }
      } else {
        const size_t prow = ((size_t)w.split * p.B * p.Hq + (size_t)w.b * p.Hq + w.h) * p.gpad + w.u0[0] + row;
        float* po = p.part_o + prow * D;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t rr[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) rr[e] = 0u;
          if (got) {
            tmem_ld32(o_addr + ch * 32, rr);
            tmem_wait_ld_dep(rr);
          }
          if (row < w.rows[0]) {
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              reinterpret_cast<float4*>(po + ch * 32)[q4] =
                  make_float4(__uint_as_float(rr[q4 * 4 + 0]) * inv, __uint_as_float(rr[q4 * 4 + 1]) * inv,
                              __uint_as_float(rr[q4 * 4 + 2]) * inv, __uint_as_float(rr[q4 * 4 + 3]) * inv);
          }
        }
        if (row < w.rows[0]) p.part_lse[prow] = got ? lse_v : -INFINITY;
      }
    } else if (MODE == 0) {
      write_zero_row<D>(p, w, x, row);
    }
  }

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

template <int D, int MODE>
static cudaError_t launch_one(const AttnParams& p, dim3 grid, cudaStream_t s) {
  auto kern = attn_tc_kernel<D, MODE>;
  const int smem = static_cast<int>(Cfg<D>::kSmemBytes);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

// p.tiles[h] holds the number of two-tile units of head h.
cudaError_t launch_band_tc(const AttnParams& p, int max_units, cudaStream_t s) {
  dim3 grid(max_units, p.Hq, p.B);
  return p.D == 64 ? launch_one<64, 0>(p, grid, s) : launch_one<128, 0>(p, grid, s);
}

cudaError_t launch_global_rows_tc(const AttnParams& p, cudaStream_t s) {
  dim3 grid(p.nsplit, p.gpad / kTile, p.B * p.Hq);
  return p.D == 64 ? launch_one<64, 1>(p, grid, s) : launch_one<128, 1>(p, grid, s);
}

}  // namespace swa
