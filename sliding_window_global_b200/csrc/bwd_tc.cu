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
//   bwd_dkv_kernel<D>    key-stationary: one CTA per 128-key tile walks the query
//                        tiles (of every query head of its GQA group) that reach
//                        it: S^T = K Q^T and dP^T = V dO^T, P^T and dS^T written
//                        back as bf16, dV += P^T dO and dK += dS^T Q.
// Neither needs atomics: every output row belongs to one CTA.  S and dP are
// computed by both passes (seven tile products instead of five), the price of
// keeping dQ out of the key-stationary pass's TMEM, which D = 128 fills.
//
// Warp roles (192 threads): warps 0-3 compute (thread t owns TMEM lane t),
// warp 4 issues the TMA loads, warp 5 allocates TMEM and issues the MMAs.
#include "ptx.cuh"
#include "swa_kernels.h"

namespace swa {
namespace {

constexpr int kBThreads = 192;
constexpr uint32_t kBSub = 128 * 128;          // one 128-row x 128-byte swizzle sub-tile
constexpr float kBLog2e = 1.4426950408889634f;

template <int D>
struct BCfg {
  static constexpr uint32_t kTileBytes = 128u * D * 2u;
  // a stationary pair of tiles, then a two-stage ring of tile pairs
  static constexpr uint32_t kStat0 = 0;
  static constexpr uint32_t kStat1 = kTileBytes;
  static constexpr uint32_t kRing = 2 * kTileBytes;   // stage s: first tile at kRing + 2 s T
  static constexpr uint32_t kStage = 512;             // lse / Delta staging (dKV): 2 x 2 x 128 floats
  static constexpr uint32_t kStageOff = kRing + 4 * kTileBytes;
  static constexpr uint32_t kBarOff = kStageOff + 4 * kStage * 4;
  static constexpr uint32_t kSmemBytes = kBarOff + 16 * 8 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  // TMEM columns: S (or S^T) 0-127 with P / dS written over 0-63; dP (or dP^T)
  // 128-255 (dS^T over 128-191 in the key-stationary pass); accumulators after.
  static constexpr uint32_t kS = 0, kDP = 128, kAcc0 = 256, kAcc1 = 256 + D;
};

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
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * kBSub + (kk & 3) * 32;
    umma_ss(dst, sdesc_sw128(a + off, 16, 1024), sdesc_sw128(b + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
  }
}

// C (+)= P X: P a 128 x 128 bf16 matrix in TMEM (packed two per column), X a
// 128 x D tile in shared memory read as an MN-major B operand.
template <int D>
__device__ __forceinline__ void mma_px(uint32_t dst, uint32_t p_tmem, uint32_t x, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, true);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    umma_ts(dst, p_tmem + kk * 8, sdesc_sw128(x + kk * 2048, kBSub, 1024), idesc,
            (accumulate || kk > 0) ? 1u : 0u);
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
__global__ void bwd_delta_kernel(const __grid_constant__ BwdParams p) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const size_t rows = (size_t)p.B * p.Hq * p.n;
  if ((size_t)warp >= rows) return;
  const __nv_bfloat16* o = static_cast<const __nv_bfloat16*>(p.out) + (size_t)warp * p.D;
  const __nv_bfloat16* g = static_cast<const __nv_bfloat16*>(p.dout) + (size_t)warp * p.D;
  float acc = 0.f;
  for (int x = lane; x < p.D; x += 32) acc = fmaf(__bfloat162float(o[x]), __bfloat162float(g[x]), acc);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) p.delta[warp] = acc;
}

// ------------------------------------------------------------------ dQ
template <int D>
__global__ void __launch_bounds__(kBThreads, 1) bwd_dq_kernel(const __grid_constant__ BwdParams p) {
  using C = BCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* a_full = bars;          // Q and dO loaded
  uint64_t* r_full = bars + 1;      // [2] K, V of a stage loaded
  uint64_t* r_empty = bars + 3;     // [2] the stage's last MMA completed
  uint64_t* s_full = bars + 5;      // S and dP in TMEM
  uint64_t* ds_full = bars + 6;     // dS written (128 arrivals)
  uint64_t* acc_full = bars + 7;    // dQ complete
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  BUnit u;
  decode_bunit(p, blockIdx.x, false, u);
  if (!u.valid) return;
  // band key range of the tile: [klo_t, khi_t) in class coordinates
  const int last = u.u0 + u.nvalid - 1;
  const int klo_t = max(0, u.u0 - u.r);
  const int khi_t = u.nvalid > 0 ? (p.causal ? min(u.Vc, last + 1) : min(u.Vc, last + u.r + 1)) : klo_t;
  const int T = khi_t > klo_t ? (khi_t - klo_t + kTile - 1) / kTile : 0;

  if (tid == 0) {
    mbar_init(a_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&r_full[s], 1);
      mbar_init(&r_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(ds_full, 128);
    mbar_init(acc_full, 1);
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
  const int qz = u.b * p.Hq + u.h;
  const int kz = u.b * p.Hkv + u.hk;

  if (warp == 4) {
    if (lane == 0 && T > 0) {
      mbar_arrive_expect_tx(a_full, 2 * C::kTileBytes);
      load_tile<D>(smem + C::kStat0, &p.mq[u.cls], a_full, u.u0, qz);
      load_tile<D>(smem + C::kStat1, &p.mdo[u.cls], a_full, u.u0, qz);
      for (int j = 0; j < T; ++j) {
        const int st = j & 1;
        if (j >= 2 && !mbar_wait_bounded(&r_empty[st], ((j >> 1) - 1) & 1, abort_v, kWaitLimitNs)) break;
        uint8_t* dst = smem + C::kRing + st * 2 * C::kTileBytes;
        mbar_arrive_expect_tx(&r_full[st], 2 * C::kTileBytes);
        load_tile<D>(dst, &p.mk[u.cls], &r_full[st], klo_t + j * kTile, kz);
        load_tile<D>(dst + C::kTileBytes, &p.mv[u.cls], &r_full[st], klo_t + j * kTile, kz);
      }
    }
  } else if (warp == 5) {
    if (lane == 0 && T > 0) {
      const uint32_t qa = smem_u32(smem + C::kStat0), da = smem_u32(smem + C::kStat1);
      bool ok = mbar_wait_bounded(a_full, 0, abort_v, kWaitLimitNs);
      for (int j = 0; ok && j <= T; ++j) {
        if (j > 0) {
          // dQ += dS(j-1) K(j-1), then the stage of tile j-1 may be refilled
          if (!mbar_wait_bounded(ds_full, (j - 1) & 1, abort_v, kWaitLimitNs)) break;
          tc_fence_after();
          const int sp = (j - 1) & 1;
          mma_px<D>(tmem + C::kAcc0, tmem + C::kS, smem_u32(smem + C::kRing + sp * 2 * C::kTileBytes), j > 1);
          umma_commit(&r_empty[sp]);
          if (j == T) umma_commit(acc_full);
        }
        if (j < T) {
          const int st = j & 1;
          if (!mbar_wait_bounded(&r_full[st], (j >> 1) & 1, abort_v, kWaitLimitNs)) break;
          tc_fence_after();
          const uint32_t kb = smem_u32(smem + C::kRing + st * 2 * C::kTileBytes);
          mma_abt<D>(tmem + C::kS, qa, kb);                          // S = Q K^T
          mma_abt<D>(tmem + C::kDP, da, kb + C::kTileBytes);         // dP = dO V^T
          umma_commit(s_full);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ compute
    const int row = tid;                       // TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const bool row_valid = row < u.nvalid;
    const int uq = u.u0 + row;
    const int klo = uq - u.r;
    const int khi = row_valid ? min(p.causal ? uq : uq + u.r, u.Vc - 1) + 1 : klo;
    size_t prow = 0;
    float lse2 = 0.f, delta = 0.f;
    if (row < u.rows) {
      prow = pos_row(p, u, u.h, p.Hq, uq);
      if (row_valid) {
        lse2 = p.lse[prow] * kBLog2e;
        delta = p.delta[prow];
      }
    }
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      if (!mbar_wait_bounded(s_full, j & 1, abort_v, kWaitLimitNs)) { ok = false; break; }
      tc_fence_after();
      const int kv0 = klo_t + j * kTile;
      const int lo_t = klo - kv0, hi_t = khi - kv0;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t sr[32], dr[32];
        tmem_ld32(lane_base + C::kS + ch * 32, sr);
        tmem_ld32(lane_base + C::kDP + ch * 32, dr);
        tmem_wait_ld_dep(sr);
        tmem_wait_ld_dep(dr);
        uint32_t pk[16];
#pragma unroll
        for (int q = 0; q < 32; q += 2) {
          float ds[2];
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int e = ch * 32 + q + h2;
            const bool allowed = e >= lo_t && e < hi_t;
            const float pr = allowed ? ex2_approx(__uint_as_float(sr[q + h2]) * sl2 - lse2) : 0.f;
            ds[h2] = pr * (__uint_as_float(dr[q + h2]) - delta);
          }
          pk[q / 2] = pack_bf16x2(ds[0], ds[1]);
        }
        // dS as bf16 over S: chunk ch writes columns 16ch.. that earlier chunks read
        tmem_st16(lane_base + C::kS + ch * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    // epilogue: dQ = scale * (dS K), fp32; padded rows get zeros
    if (ok && T > 0) ok = mbar_wait_bounded(acc_full, 0, abort_v, kWaitLimitNs);
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
        if (row < u.rows) {
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (T > 0 && row_valid)
              v4 = make_float4(__uint_as_float(rr[q4 * 4]) * p.scale, __uint_as_float(rr[q4 * 4 + 1]) * p.scale,
                               __uint_as_float(rr[q4 * 4 + 2]) * p.scale, __uint_as_float(rr[q4 * 4 + 3]) * p.scale);
            reinterpret_cast<float4*>(dst)[ch * 8 + q4] = v4;
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
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------------ dK, dV
template <int D>
__global__ void __launch_bounds__(kBThreads, 1) bwd_dkv_kernel(const __grid_constant__ BwdParams p) {
  using C = BCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  float* sStage = reinterpret_cast<float*>(smem + C::kStageOff);   // [2][lse2, delta][128]
  uint64_t* a_full = bars;          // K and V loaded
  uint64_t* r_full = bars + 1;      // [2] Q, dO of a stage loaded
  uint64_t* r_empty = bars + 3;     // [2]
  uint64_t* s_full = bars + 5;      // S^T and dP^T in TMEM
  uint64_t* p_full = bars + 6;      // P^T and dS^T written (128 arrivals)
  uint64_t* acc_full = bars + 7;    // dK, dV complete
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  BUnit u;
  decode_bunit(p, blockIdx.x, true, u);
  if (!u.valid) return;
  // query rows (class coordinates) whose window reaches the valid keys of this tile
  const int lastk = u.u0 + u.nvalid - 1;
  const int qlo = p.causal ? u.u0 : max(0, u.u0 - u.r);
  const int qhi = u.nvalid > 0 ? min(u.Vc, lastk + u.r + 1) : qlo;
  const int NQ = qhi > qlo ? (qhi - qlo + kTile - 1) / kTile : 0;
  const int T = NQ * p.G;                     // query tiles of every head of the group

  if (tid == 0) {
    mbar_init(a_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&r_full[s], 1);
      mbar_init(&r_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(acc_full, 1);
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
  const int kz = u.b * p.Hkv + u.hk;

  if (warp == 4) {
    if (lane == 0 && T > 0) {
      mbar_arrive_expect_tx(a_full, 2 * C::kTileBytes);
      load_tile<D>(smem + C::kStat0, &p.mk[u.cls], a_full, u.u0, kz);
      load_tile<D>(smem + C::kStat1, &p.mv[u.cls], a_full, u.u0, kz);
      for (int j = 0; j < T; ++j) {
        const int st = j & 1;
        if (j >= 2 && !mbar_wait_bounded(&r_empty[st], ((j >> 1) - 1) & 1, abort_v, kWaitLimitNs)) break;
        const int qz = u.b * p.Hq + u.h + j / NQ;
        const int y = qlo + (j % NQ) * kTile;
        uint8_t* dst = smem + C::kRing + st * 2 * C::kTileBytes;
        mbar_arrive_expect_tx(&r_full[st], 2 * C::kTileBytes);
        load_tile<D>(dst, &p.mq[u.cls], &r_full[st], y, qz);
        load_tile<D>(dst + C::kTileBytes, &p.mdo[u.cls], &r_full[st], y, qz);
      }
    }
  } else if (warp == 5) {
    if (lane == 0 && T > 0) {
      const uint32_t ka = smem_u32(smem + C::kStat0), va = smem_u32(smem + C::kStat1);
      bool ok = mbar_wait_bounded(a_full, 0, abort_v, kWaitLimitNs);
      for (int j = 0; ok && j <= T; ++j) {
        if (j > 0) {
          // dV += P^T dO and dK += dS^T Q for tile j-1, then its stage may be refilled
          if (!mbar_wait_bounded(p_full, (j - 1) & 1, abort_v, kWaitLimitNs)) break;
          tc_fence_after();
          const int sp = (j - 1) & 1;
          const uint32_t qb = smem_u32(smem + C::kRing + sp * 2 * C::kTileBytes);
          mma_px<D>(tmem + C::kAcc0, tmem + C::kS, qb + C::kTileBytes, j > 1);   // dV
          mma_px<D>(tmem + C::kAcc1, tmem + C::kDP, qb, j > 1);                  // dK
          umma_commit(&r_empty[sp]);
          if (j == T) umma_commit(acc_full);
        }
        if (j < T) {
          const int st = j & 1;
          if (!mbar_wait_bounded(&r_full[st], (j >> 1) & 1, abort_v, kWaitLimitNs)) break;
          tc_fence_after();
          const uint32_t qb = smem_u32(smem + C::kRing + st * 2 * C::kTileBytes);
          mma_abt<D>(tmem + C::kS, ka, qb);                          // S^T = K Q^T
          mma_abt<D>(tmem + C::kDP, va, qb + C::kTileBytes);         // dP^T = V dO^T
          umma_commit(s_full);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ compute
    const int row = tid;                       // key row, TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const bool key_valid = row < u.nvalid;
    const int uk = u.u0 + row;
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      // stage lse2 and Delta of the tile's 128 query rows (a padded or missing row
      // gets lse2 = +inf, so its p is 0)
      const int head = u.h + j / NQ;
      const int q0 = qlo + (j % NQ) * kTile;
      float* stg = sStage + (j & 1) * 256;
      {
        const int uq = q0 + row;
        float l2 = INFINITY, dl = 0.f;
        if (uq < u.Vc) {
          const size_t pr = pos_row(p, u, head, p.Hq, uq);
          l2 = p.lse[pr] * kBLog2e;
          dl = p.delta[pr];
        }
        stg[row] = l2;
        stg[128 + row] = dl;
      }
      named_barrier_sync(1, 128);
      if (!mbar_wait_bounded(s_full, j & 1, abort_v, kWaitLimitNs)) { ok = false; break; }
      tc_fence_after();
      const int d0 = q0 - uk;                  // query - key offset of column 0
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t sr[32], dr[32];
        tmem_ld32(lane_base + C::kS + ch * 32, sr);
        tmem_ld32(lane_base + C::kDP + ch * 32, dr);
        tmem_wait_ld_dep(sr);
        tmem_wait_ld_dep(dr);
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int q = 0; q < 32; q += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(stg + ch * 32 + q);
          const float4 dl4 = *reinterpret_cast<const float4*>(stg + 128 + ch * 32 + q);
          const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
          const float dv[4] = {dl4.x, dl4.y, dl4.z, dl4.w};
          float pr[4], ds[4];
#pragma unroll
          for (int e4 = 0; e4 < 4; ++e4) {
            const int off = d0 + ch * 32 + q + e4;   // query - key
            const bool inband = p.causal ? (off >= 0 && off <= u.r) : (off >= -u.r && off <= u.r);
            const bool allowed = key_valid && inband;
            pr[e4] = allowed ? ex2_approx(__uint_as_float(sr[q + e4]) * sl2 - lv[e4]) : 0.f;
            ds[e4] = pr[e4] * (__uint_as_float(dr[q + e4]) - dv[e4]);
          }
          pk[q / 2] = pack_bf16x2(pr[0], pr[1]);
          pk[q / 2 + 1] = pack_bf16x2(pr[2], pr[3]);
          dk[q / 2] = pack_bf16x2(ds[0], ds[1]);
          dk[q / 2 + 1] = pack_bf16x2(ds[2], ds[3]);
        }
        tmem_st16(lane_base + C::kS + ch * 16, pk);     // P^T over S^T
        tmem_st16(lane_base + C::kDP + ch * 16, dk);    // dS^T over dP^T
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    // epilogue: dK = scale * (dS^T Q), dV = P^T dO, fp32; padded keys get zeros.
    // The TMEM loads are warp-wide, so every thread issues them; only rows of the
    // tile store.
    if (ok && T > 0) ok = mbar_wait_bounded(acc_full, 0, abort_v, kWaitLimitNs);
    if (ok) {
      tc_fence_after();
      const size_t prow = row < u.rows ? pos_row(p, u, u.hk, p.Hkv, uk) : 0;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        float* dst = (which ? p.dk : p.dv) + prow * D;
        const float mul = which ? p.scale : 1.f;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t rr[32];
          if (T > 0) {
            tmem_ld32(lane_base + (which ? C::kAcc1 : C::kAcc0) + ch * 32, rr);
            tmem_wait_ld_dep(rr);
          }
          if (row < u.rows) {
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
              float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
              if (T > 0 && key_valid)
                v4 = make_float4(__uint_as_float(rr[q4 * 4]) * mul, __uint_as_float(rr[q4 * 4 + 1]) * mul,
                                 __uint_as_float(rr[q4 * 4 + 2]) * mul, __uint_as_float(rr[q4 * 4 + 3]) * mul);
              reinterpret_cast<float4*>(dst)[ch * 8 + q4] = v4;
            }
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
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <typename K>
cudaError_t launch_bwd(K kern, uint32_t smem, int grid, const BwdParams& p, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (grid <= 0) return cudaSuccess;
  kern<<<grid, kBThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_delta(const BwdParams& p, cudaStream_t s) {
  const size_t rows = (size_t)p.B * p.Hq * p.n;
  const int blocks = (int)((rows * 32 + 255) / 256);
  bwd_delta_kernel<<<blocks, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dq(const BwdParams& p, cudaStream_t s) {
  const int grid = p.max_qtiles * p.B * p.Hq;
  return p.D == 64 ? launch_bwd(bwd_dq_kernel<64>, BCfg<64>::kSmemBytes, grid, p, s)
                   : launch_bwd(bwd_dq_kernel<128>, BCfg<128>::kSmemBytes, grid, p, s);
}

cudaError_t launch_bwd_dkv(const BwdParams& p, cudaStream_t s) {
  const int grid = p.max_ktiles * p.B * p.Hkv;
  return p.D == 64 ? launch_bwd(bwd_dkv_kernel<64>, BCfg<64>::kSmemBytes, grid, p, s)
                   : launch_bwd(bwd_dkv_kernel<128>, BCfg<128>::kSmemBytes, grid, p, s);
}

}  // namespace swa
