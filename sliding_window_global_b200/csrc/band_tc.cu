// band_tc.cu -- tcgen05 (5th-generation tensor core) kernel for banded sparse
// self-attention on sm_100a, bf16 inputs with fp32 accumulation in TMEM.
//
// One CTA owns one tile of 128 query rows of one (batch, query head, residue
// class) and walks a list of 128-key tiles:
//   band tiles   -- keys of the (dilated, optionally causal) sliding window
//                   (BigBird notes §3.2.1; Longformer page §二 for dilation;
//                   SWAN-GPT §3.3(1) for the causal 512-key window), only the
//                   tiles the window touches, so fully masked tiles are skipped;
//   global tiles -- the gathered global tokens every query also attends to,
//                   minus those already inside its window (BigBird §3.2.3 ITC);
//   side tiles   -- appended side keys with the additive bucketed bias of the
//                   LongT5 Transient-Global attention ("LongT5 长序列模型完全指南",
//                   Local / Transient-Global and 源码级证据 sections).
// With dilation d a query at position c + d*u only meets keys c + d*u', so the
// kernel works in residue-class coordinates: every class is a plain band of
// radius r over rows c, c+d, ..., loaded through a strided TMA tensor map.
//
// The same kernel in MODE 1 computes global query rows (full attention over all
// valid keys plus side keys) split over key ranges; a merge kernel combines the
// splits by logsumexp and overwrites those rows.
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread t owns query row t (TMEM lane t): loads S from
//              TMEM, masks, scales, adds bias, online softmax (running max m and
//              sum l, lazy O rescale), writes P (bf16) to shared memory, and
//              finally normalises O and stores it;
//   warp 4     TMA producer: Q once, then K/V tiles into an NS-stage ring;
//   warp 5     TMEM allocator and MMA issuer: S = Q K^T into one of two TMEM
//              S buffers, O += P V into the TMEM O accumulator.
#include "ptx.cuh"
#include "swa_kernels.h"

namespace swa {
namespace {

constexpr int kThreads = 192;
constexpr uint32_t kSub = 128 * 128;          // one 128-row x 128-byte swizzle sub-tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;     // log2 units: rescale O only when max grows > 2^8

template <int D>
struct Cfg {
  static constexpr int NS = (D == 64) ? 3 : 2;                 // K/V ring stages
  static constexpr uint32_t kTileBytes = 128u * D * 2u;        // one 128 x D bf16 tile
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKOff = kQOff + kTileBytes;
  static constexpr uint32_t kVOff = kKOff + NS * kTileBytes;
  static constexpr uint32_t kPOff = kVOff + NS * kTileBytes;
  static constexpr uint32_t kBarOff = kPOff + 2 * kSub;        // P: 128 x 128 bf16
  static constexpr int kNumBars = 1 + 3 * NS + 2 + 2 + 1 + 1;
  static constexpr uint32_t kSmemBytes = kBarOff + kNumBars * 8 + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = 512;                    // S0 | S1 | O
  static constexpr uint32_t kOCol = 256;
};

struct TileList {
  int nband, ngc, nside, total;
  int band_lo;          // first key (class coordinates) of band tile 0
  int key_end;          // band keys at or beyond this are masked (global-row split end)
  int map_class;        // class whose K/V maps the band tiles use
};

// Per-CTA work description, identical in every thread.
struct Work {
  int b, h, hk;
  int cls;              // residue class of the query rows (MODE 0)
  int u0;               // first query row of the tile (class coordinates / global slot)
  int rows;             // rows of this tile that exist (<= 128)
  int valid_rows;       // rows below the valid length (MODE 0) / below g (MODE 1)
  int Vc;               // valid rows of the class (MODE 0) / valid keys (MODE 1)
  int split;            // MODE 1: key split index
  int d, c, r;
  bool active;          // false: no key work at all
  TileList t;
};

template <int MODE>
__device__ __forceinline__ bool decode_work(const AttnParams& p, Work& w) {
  if (MODE == 0) {
    w.b = blockIdx.z;
    w.h = blockIdx.y;
    int tile = blockIdx.x;
    if (tile >= p.tiles[w.h]) return false;
    w.hk = w.h / p.G;
    w.r = p.window[w.h];
    int base = p.class_base[w.h];
    w.d = p.cls[base].d;
    int c = 0;
    for (; c < w.d; ++c) {
      int tc = (p.cls[base + c].n_c + kTile - 1) / kTile;
      if (tile < tc) break;
      tile -= tc;
    }
    w.c = c;
    w.cls = base + c;
    int nc = p.cls[w.cls].n_c;
    int V = p.valid_len ? p.valid_len[w.b] : p.n;
    if (V > p.n) V = p.n;
    w.Vc = V > c ? (V - c + w.d - 1) / w.d : 0;
    w.u0 = tile * kTile;
    w.rows = min(kTile, nc - w.u0);
    w.valid_rows = max(0, min(w.rows, w.Vc - w.u0));
    w.split = 0;
    w.active = w.valid_rows > 0;
    TileList& t = w.t;
    t.map_class = w.cls;
    t.band_lo = max(0, w.u0 - w.r);
    int hi = p.causal ? min(w.Vc, w.u0 + kTile) : min(w.Vc, w.u0 + kTile - 1 + w.r + 1);
    t.nband = w.active ? (hi - t.band_lo + kTile - 1) / kTile : 0;
    t.key_end = hi;
    t.ngc = (w.active && p.g > 0) ? (p.g + kTile - 1) / kTile : 0;
    t.nside = (w.active && p.S > 0) ? (p.S + kTile - 1) / kTile : 0;
    t.total = t.nband + t.ngc + t.nside;
  } else {
    w.split = blockIdx.x;
    int gt = blockIdx.y;
    int bh = blockIdx.z;
    w.b = bh / p.Hq;
    w.h = bh % p.Hq;
    w.hk = w.h / p.G;
    w.r = 0;
    w.d = 1;
    w.c = 0;
    w.cls = p.dense_class;
    int V = p.valid_len ? p.valid_len[w.b] : p.n;
    if (V > p.n) V = p.n;
    w.Vc = V;
    w.u0 = gt * kTile;
    w.rows = min(kTile, p.gpad - w.u0);
    w.valid_rows = max(0, min(w.rows, p.g - w.u0));
    TileList& t = w.t;
    t.map_class = p.dense_class;
    t.ngc = 0;
    if (w.split < p.nsplit_keys) {
      int k0 = w.split * p.split_keys;
      int k1 = min(V, k0 + p.split_keys);
      t.band_lo = k0;
      t.key_end = k1;
      t.nband = (k1 > k0) ? (k1 - k0 + kTile - 1) / kTile : 0;
      t.nside = 0;
    } else {
      t.band_lo = 0;
      t.key_end = 0;
      t.nband = 0;
      t.nside = (p.S + kTile - 1) / kTile;
    }
    w.active = w.valid_rows > 0 && (t.nband + t.nside) > 0;
    if (!w.active) t.nband = t.nside = 0;
    t.total = t.nband + t.ngc + t.nside;
  }
  return true;
}

// Which maps and coordinates tile j uses.
__device__ __forceinline__ void tile_source(const AttnParams& p, const Work& w, int j,
                                            const CUtensorMap*& mk, const CUtensorMap*& mv,
                                            int& y) {
  const TileList& t = w.t;
  if (j < t.nband) {
    mk = &p.mk[t.map_class];
    mv = &p.mv[t.map_class];
    y = t.band_lo + j * kTile;
  } else if (j < t.nband + t.ngc) {
    mk = &p.mgk;
    mv = &p.mgv;
    y = (j - t.nband) * kTile;
  } else {
    mk = &p.msk;
    mv = &p.msv;
    y = (j - t.nband - t.ngc) * kTile;
  }
}

template <int D>
__device__ __forceinline__ void tma_tile(void* dst, const CUtensorMap* map, uint64_t* bar, int y,
                                         int z) {
  tma_load_3d(dst, map, bar, 0, y, z);
  if (D == 128) tma_load_3d(static_cast<uint8_t*>(dst) + kSub, map, bar, 64, y, z);
}

// Rows of this CTA that are padding (MODE 0) get o = 0 and lse = -inf.
template <int D>
__device__ void write_padding_rows(const AttnParams& p, const Work& w, int row) {
  if (row >= w.rows || row < w.valid_rows) return;
  int pos = w.c + w.d * (w.u0 + row);
  size_t off = ((size_t)(w.b * p.Hq + w.h) * p.n + pos);
  uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + off * D);
#pragma unroll
  for (int x = 0; x < D / 8; ++x) o[x] = make_uint4(0, 0, 0, 0);
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
  uint8_t* sP = smem + C::kPOff;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + NS;
  uint64_t* kv_empty = v_full + NS;
  uint64_t* s_full = kv_empty + NS;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* o_done = p_full + 1;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  Work w;
  if (!decode_work<MODE>(p, w)) return;

  if (!w.active) {
    if (MODE == 0) {
      if (tid < kTile) write_padding_rows<D>(p, w, tid);
    } else if (tid < kTile) {
      // empty split: neutral partial (o = 0, lse = -inf)
      int slot = w.u0 + tid;
      if (slot < p.gpad) {
        size_t prow = ((size_t)w.split * p.B * p.Hq + (size_t)w.b * p.Hq + w.h) * p.gpad + slot;
        float4* po = reinterpret_cast<float4*>(p.part_o + prow * D);
        for (int x = 0; x < D / 4; ++x) po[x] = make_float4(0.f, 0.f, 0.f, 0.f);
        p.part_lse[prow] = -INFINITY;
      }
    }
    return;
  }

  const int T = w.t.total;

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_free[s], kTile);
    }
    mbar_init(p_full, kTile);
    mbar_init(o_done, 1);
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

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const CUtensorMap* mq = (MODE == 0) ? &p.mq[w.cls] : &p.mgq;
      tma_prefetch_desc(mq);
      const int qz = w.b * p.Hq + w.h;
      const int kz = w.b * p.Hkv + w.hk;
      mbar_arrive_expect_tx(q_full, C::kTileBytes);
      tma_tile<D>(sQ, mq, q_full, w.u0, qz);
      for (int j = 0; j < T; ++j) {
        const int st = j % NS;
        const int use = j / NS;
        if (j >= NS && !mbar_wait_bounded(&kv_empty[st], (use - 1) & 1, abort_v, kWaitLimitNs))
          break;
        const CUtensorMap *mk, *mv;
        int y;
        tile_source(p, w, j, mk, mv, y);
        mbar_arrive_expect_tx(&k_full[st], C::kTileBytes);
        tma_tile<D>(sK + st * C::kTileBytes, mk, &k_full[st], y, kz);
        mbar_arrive_expect_tx(&v_full[st], C::kTileBytes);
        tma_tile<D>(sV + st * C::kTileBytes, mv, &v_full[st], y, kz);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t k_base = smem_u32(sK);
      const uint32_t v_base = smem_u32(sV);
      const uint32_t p_base = smem_u32(sP);
      bool ok = mbar_wait_bounded(q_full, 0, abort_v, kWaitLimitNs);
      auto issue_pv = [&](int jj) -> bool {
        const int st = jj % NS;
        if (!mbar_wait_bounded(p_full, jj & 1, abort_v, kWaitLimitNs)) return false;
        if (!mbar_wait_bounded(&v_full[st], (jj / NS) & 1, abort_v, kWaitLimitNs)) return false;
        tc_fence_after();
        const uint32_t vt = v_base + st * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          uint64_t a = sdesc_sw128(p_base + (kk >> 2) * kSub + (kk & 3) * 32, 16, 1024);
          uint64_t b = sdesc_sw128(vt + kk * 2048, kSub, 1024);
          umma_ss(tmem + C::kOCol, a, b, idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&kv_empty[st]);
        umma_commit(o_done);
        return true;
      };
      for (int j = 0; ok && j < T; ++j) {
        const int st = j % NS;
        const int sb = j & 1;
        if (!mbar_wait_bounded(&k_full[st], (j / NS) & 1, abort_v, kWaitLimitNs)) { ok = false; break; }
        if (j >= 2 && !mbar_wait_bounded(&s_free[sb], ((j >> 1) - 1) & 1, abort_v, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kt = k_base + st * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kSub + (kk & 3) * 32;
          uint64_t a = sdesc_sw128(q_base + off, 16, 1024);
          uint64_t b = sdesc_sw128(kt + off, 16, 1024);
          umma_ss(tmem + sb * 128, a, b, idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[sb]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) issue_pv(T - 1);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int row = tid;                       // TMEM lane == query row in the tile
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    const bool row_valid = row < w.valid_rows;
    int pos = 0;                               // sequence position of this query row
    if (MODE == 0) {
      pos = w.c + w.d * (w.u0 + row);
    } else if (row_valid) {
      pos = p.global_idx[(size_t)w.b * p.g + w.u0 + row];
    }
    const int u = w.u0 + row;                  // class coordinate (MODE 0)
    const int rd = w.r * w.d;
    const int qblk = (p.S > 0) ? pos / p.side_block : 0;
    const float* bias_row =
        (p.bias && p.S > 0) ? p.bias + (size_t)w.h * (p.S + p.nblk - 1) + (p.nblk - 1 - qblk) : nullptr;
    float m = -INFINITY;                       // running max (log2 units)
    float l = 0.f;                             // running sum
    bool ok = true;

    for (int j = 0; j < T; ++j) {
      const int sb = j & 1;
      if (!mbar_wait_bounded(&s_full[sb], (j >> 1) & 1, abort_v, kWaitLimitNs)) { ok = false; break; }
      tc_fence_after();
      uint32_t xr[kTile];
#pragma unroll
      for (int ch = 0; ch < 4; ++ch)
        tmem_ld32(lane_addr + sb * 128 + ch * 32, *reinterpret_cast<uint32_t(*)[32]>(xr + ch * 32));
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) tmem_wait_ld_dep(*reinterpret_cast<uint32_t(*)[32]>(xr + ch * 32));
      float x[kTile];
#pragma unroll
      for (int e = 0; e < kTile; ++e) x[e] = __uint_as_float(xr[e]);
      tc_fence_before();
      mbar_arrive(&s_free[sb]);

      // mask, scale, bias -> x in log2 units; masked entries -inf
      float tmax = -INFINITY;
      if (j < w.t.nband) {
        const int kv0 = w.t.band_lo + j * kTile;
        int lo_t, hi_t;
        if (MODE == 0) {
          lo_t = u - w.r - kv0;
          hi_t = min(p.causal ? u : u + w.r, w.Vc - 1) + 1 - kv0;
        } else {
          lo_t = 0;
          hi_t = w.t.key_end - kv0;
        }
        if (!row_valid) hi_t = lo_t;           // padded query row: nothing attended
#pragma unroll
        for (int e = 0; e < kTile; ++e) {
          float v = x[e] * p.scale_log2;
          v = (e >= lo_t && e < hi_t) ? v : -INFINITY;
          x[e] = v;
          tmax = fmaxf(tmax, v);
        }
      } else if (j < w.t.nband + w.t.ngc) {
        const int e0 = (j - w.t.nband) * kTile;
        const int32_t* gl = p.global_idx + (size_t)w.b * p.g;
#pragma unroll
        for (int e = 0; e < kTile; ++e) {
          bool allowed = false;
          if (row_valid && e0 + e < p.g) {
            int diff = pos - __ldg(gl + e0 + e);
            bool inwin = p.causal ? (diff >= 0 && diff <= rd) : (abs(diff) <= rd);
            inwin = inwin && (diff % w.d == 0);
            allowed = !inwin;
          }
          float v = allowed ? x[e] * p.scale_log2 : -INFINITY;
          x[e] = v;
          tmax = fmaxf(tmax, v);
        }
      } else {
        const int s0 = (j - w.t.nband - w.t.ngc) * kTile;
        const int lim = row_valid ? p.S - s0 : 0;
#pragma unroll
        for (int e = 0; e < kTile; ++e) {
          float v = -INFINITY;
          if (e < lim) {
            float bb = bias_row ? __ldg(bias_row + s0 + e) : 0.f;
            v = x[e] * p.scale_log2 + bb * kLog2e;
          }
          x[e] = v;
          tmax = fmaxf(tmax, v);
        }
      }

      // P buffer free and O stable once the previous PV has completed
      if (j > 0 && !mbar_wait_bounded(o_done, (j - 1) & 1, abort_v, kWaitLimitNs)) { ok = false; break; }
      tc_fence_after();
      const float m_new = fmaxf(m, tmax);
      const bool need = (m == -INFINITY) ? (m_new > -INFINITY) : (m_new > m + kRescaleThreshold);
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = (m == -INFINITY) ? 0.f : ex2_approx(m - m_new);
        if (j > 0) {
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t rr[32];
            tmem_ld32(lane_addr + C::kOCol + ch * 32, rr);
            tmem_wait_ld_dep(rr);
#pragma unroll
            for (int e = 0; e < 32; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * alpha);
            tmem_st32(lane_addr + C::kOCol + ch * 32, rr);
          }
          tmem_wait_st();
        }
        l *= alpha;
        m = m_new;
      }
      const float mref = (m == -INFINITY) ? 0.f : m;
      float lsum = 0.f;
#pragma unroll
      for (int sub = 0; sub < 2; ++sub) {
        uint8_t* prow = sP + sub * kSub + row * 128;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          const int e = sub * 64 + c8 * 8;
          float p0 = ex2_approx(x[e + 0] - mref), p1 = ex2_approx(x[e + 1] - mref);
          float p2 = ex2_approx(x[e + 2] - mref), p3 = ex2_approx(x[e + 3] - mref);
          float p4 = ex2_approx(x[e + 4] - mref), p5 = ex2_approx(x[e + 5] - mref);
          float p6 = ex2_approx(x[e + 6] - mref), p7 = ex2_approx(x[e + 7] - mref);
          lsum += ((p0 + p1) + (p2 + p3)) + ((p4 + p5) + (p6 + p7));
          uint4 pk = make_uint4(pack_bf16x2(p0, p1), pack_bf16x2(p2, p3), pack_bf16x2(p4, p5),
                                pack_bf16x2(p6, p7));
          *reinterpret_cast<uint4*>(prow + ((c8 ^ (row & 7)) << 4)) = pk;
        }
      }
      l += lsum;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }

    if (ok && mbar_wait_bounded(o_done, (T - 1) & 1, abort_v, kWaitLimitNs)) {
      tc_fence_after();
      const bool has = row_valid && l > 0.f;
      const float inv = has ? 1.f / l : 0.f;
      const float lse_v = has ? (m + __log2f(l)) * kLn2 : -INFINITY;
      if (MODE == 0) {
        const size_t off = ((size_t)(w.b * p.Hq + w.h) * p.n + pos);
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + off * D;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t rr[32];
          tmem_ld32(lane_addr + C::kOCol + ch * 32, rr);
          tmem_wait_ld_dep(rr);
          if (row < w.rows) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 0]) * inv, __uint_as_float(rr[q4 * 8 + 1]) * inv);
              v.y = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 2]) * inv, __uint_as_float(rr[q4 * 8 + 3]) * inv);
              v.z = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 4]) * inv, __uint_as_float(rr[q4 * 8 + 5]) * inv);
              v.w = pack_bf16x2(__uint_as_float(rr[q4 * 8 + 6]) * inv, __uint_as_float(rr[q4 * 8 + 7]) * inv);
              reinterpret_cast<uint4*>(orow + ch * 32)[q4] = v;
            }
          }
        }
        if (row < w.rows && p.lse) p.lse[off] = lse_v;
      } else {
        const size_t prow =
            ((size_t)w.split * p.B * p.Hq + (size_t)w.b * p.Hq + w.h) * p.gpad + w.u0 + row;
        float* po = p.part_o + prow * D;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t rr[32];
          tmem_ld32(lane_addr + C::kOCol + ch * 32, rr);
          tmem_wait_ld_dep(rr);
          if (row < w.rows) {
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              reinterpret_cast<float4*>(po + ch * 32)[q4] =
                  make_float4(__uint_as_float(rr[q4 * 4 + 0]) * inv, __uint_as_float(rr[q4 * 4 + 1]) * inv,
                              __uint_as_float(rr[q4 * 4 + 2]) * inv, __uint_as_float(rr[q4 * 4 + 3]) * inv);
          }
        }
        if (row < w.rows) p.part_lse[prow] = lse_v;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (abort_flag) {
    // A bounded wait expired somewhere: report it, then give copies and MMAs
    // still in flight time to land before TMEM and shared memory are released.
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

cudaError_t launch_band_tc(const AttnParams& p, int max_tiles, cudaStream_t s) {
  dim3 grid(max_tiles, p.Hq, p.B);
  return p.D == 64 ? launch_one<64, 0>(p, grid, s) : launch_one<128, 0>(p, grid, s);
}

cudaError_t launch_global_rows_tc(const AttnParams& p, cudaStream_t s) {
  dim3 grid(p.nsplit, p.gpad / kTile, p.B * p.Hq);
  return p.D == 64 ? launch_one<64, 1>(p, grid, s) : launch_one<128, 1>(p, grid, s);
}

}  // namespace swa
