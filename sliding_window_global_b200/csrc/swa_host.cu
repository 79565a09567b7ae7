// swa_host.cu -- host set-up shared by every forward entry point (see swa_host.h).
//
// Launch sequence of one forward pass (all on the caller's stream):
//   bf16:  [debug: check global_idx / random blocks, synchronise, stop on failure]
//          -> [g > 0: gather global q/k/v rows]
//          -> band kernel (window + global columns + side keys + random blocks)
//          -> [g > 0: global-row kernel (split over keys) -> logsumexp merge that
//             overwrites the global query rows]
//   fp32:  [debug check] -> CUDA-core kernel (all rows, global rows included)
#include "swa_host.h"

#include <math.h>
#include <string.h>

#include <algorithm>

namespace swa {
namespace {

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

}  // namespace

bool make_map(CUtensorMap* m, const void* base, int D, uint64_t rows, uint64_t planes,
              uint64_t row_stride_bytes, uint64_t plane_stride_bytes, bool store_box, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows == 0 || planes == 0) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, rows, planes};
  cuuint64_t strides[2] = {row_stride_bytes, plane_stride_bytes};
  cuuint32_t box[3] = {store_box ? 32u : 64u, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  store_box ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

swa_status validate_desc(const swa_plan_desc& d) {
  if (d.batch < 1 || d.seq_len < 1 || d.num_q_heads < 1 || d.num_kv_heads < 1 ||
      d.num_q_heads % d.num_kv_heads != 0 || d.max_global < 0 || d.num_side < 0 ||
      d.head_dim < 1 || (d.dtype != SWA_BF16 && d.dtype != SWA_FP32) || d.scale < 0.f ||
      !(d.scale == d.scale) || (d.num_side > 0 && d.side_block < 1) ||
      d.max_global > d.seq_len || (d.flags & ~SWA_DEBUG_CHECKS))
    return SWA_ERR_INVALID_ARG;
  if (d.head_dim != 64 && d.head_dim != 128) return SWA_ERR_UNSUPPORTED;
  if (d.num_q_heads > kMaxHeads) return SWA_ERR_UNSUPPORTED;
  if ((long long)d.batch * d.num_q_heads > 65535LL * 65535LL) return SWA_ERR_UNSUPPORTED;
  return SWA_OK;
}

int max_global_splits(const swa_plan_desc& d) {
  const int ntiles = (d.seq_len + kTile - 1) / kTile;
  return std::min(ntiles, 64) + (d.num_side > 0 ? 1 : 0);
}

GlobalLayout global_layout(const swa_plan_desc& d, int gpad, int nsplit, size_t base) {
  const size_t B = d.batch, Hq = d.num_q_heads, Hkv = d.num_kv_heads, D = d.head_dim;
  GlobalLayout L;
  L.gq = align_up(base, 256);
  L.gk = align_up(L.gq + B * Hq * gpad * D * 2, 256);
  L.gv = align_up(L.gk + B * Hkv * gpad * D * 2, 256);
  L.po = align_up(L.gv + B * Hkv * gpad * D * 2, 256);
  L.pl = align_up(L.po + (size_t)nsplit * B * Hq * gpad * D * 4, 256);
  L.end = align_up(L.pl + (size_t)nsplit * B * Hq * gpad * 4, 256);
  return L;
}

size_t side_buffer_bytes(const swa_plan_desc& d) {
  if (d.num_side <= 0 || d.side_block < 1 || d.num_side != d.seq_len / d.side_block) return 0;
  const size_t es = d.dtype == SWA_FP32 ? 4 : 2;
  return align_up((size_t)d.batch * d.num_kv_heads * d.num_side * d.head_dim * es, 256);
}

swa_status read_and_clear_error(int* err, cudaStream_t s) {
  if (cudaStreamSynchronize(s) != cudaSuccess) return SWA_ERR_CUDA;
  int h = 0;
  if (cudaMemcpy(&h, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SWA_ERR_CUDA;
  if (h && cudaMemset(err, 0, sizeof(int)) != cudaSuccess) return SWA_ERR_CUDA;
  if (h & kDevErrTimeout) return SWA_ERR_TIMEOUT;
  if (h & kDevErrCheck) return SWA_ERR_DEVICE_CHECK;
  return SWA_OK;
}

swa_status enqueue_forward(const swa_plan_desc& d, const swa_forward_args& args,
                           const ForwardScratch& ws, int num_sms, cudaStream_t s, int* launches_out) {
  *launches_out = 0;
  const void *q = args.q, *k = args.k, *v = args.v;
  const int32_t* global_idx = args.global_idx;
  const int num_global = args.num_global;
  const void *side_k = args.side_k, *side_v = args.side_v;
  const float* bias = args.bias;
  const int32_t *window = args.window, *dilation = args.dilation;
  const int causal = args.causal;
  const int32_t* valid_len = args.valid_len;
  void* out = args.out;
  float* lse = args.lse;
  const float* local_bias = args.local_bias;
  const int32_t* rand_blocks = args.num_rand > 0 ? args.rand_blocks : nullptr;
  // ---------------------------------------------------------- validation
  if (!q || !k || !v || !out || !window || !ws.err) return SWA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SWA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SWA_ERR_INVALID_ARG;
  if (num_global < 0 || num_global > d.max_global) return SWA_ERR_INVALID_ARG;
  if (num_global > 0 && !global_idx) return SWA_ERR_INVALID_ARG;
  if (args.side_from_kv != 0 && args.side_from_kv != 1) return SWA_ERR_INVALID_ARG;
  const bool build_side = args.side_from_kv == 1;
  if (build_side) {
    // side keys / values are the block means of k and v, made here
    if (side_k || side_v || d.num_side < 1 || d.num_side != d.seq_len / d.side_block)
      return SWA_ERR_INVALID_ARG;
    if (!ws.side_k || !ws.side_v) return SWA_ERR_UNSUPPORTED;
    side_k = ws.side_k;
    side_v = ws.side_v;
  }
  if (d.num_side > 0) {
    if (!side_k || !side_v) return SWA_ERR_INVALID_ARG;
    if (!aligned16(side_k) || !aligned16(side_v)) return SWA_ERR_INVALID_ARG;
  }
  if ((lse && !aligned4(lse)) || (bias && !aligned4(bias)) || (local_bias && !aligned4(local_bias)) ||
      (rand_blocks && !aligned4(rand_blocks)) || (global_idx && !aligned4(global_idx)) ||
      (valid_len && !aligned4(valid_len)))
    return SWA_ERR_INVALID_ARG;
  if (args.num_rand < 0 || args.num_rand > kMaxRand) return SWA_ERR_INVALID_ARG;
  if (args.num_rand > 0 && !rand_blocks) return SWA_ERR_INVALID_ARG;
  const int Hq = d.num_q_heads;
  for (int h = 0; h < Hq; ++h) {
    if (window[h] < 0) return SWA_ERR_INVALID_ARG;
    if (dilation && dilation[h] < 1) return SWA_ERR_INVALID_ARG;
    if ((long long)window[h] * (dilation ? dilation[h] : 1) > (1LL << 30)) return SWA_ERR_INVALID_ARG;
  }
  if (causal && num_global > 0) return SWA_ERR_UNSUPPORTED;
  if (rand_blocks) {
    // random key blocks are tiles of the plain key sequence: dilation 1, non-causal
    if (causal) return SWA_ERR_UNSUPPORTED;
    for (int h = 0; h < Hq; ++h)
      if (dilation && dilation[h] != 1) return SWA_ERR_UNSUPPORTED;
  }
  // local bias: the table covers every offset a window key can take; the band
  // kernel stages [-r_eff - kLocalPad, r_eff + kLocalPad] of it per work unit,
  // r_eff = min(r, ceil(n / d)) (offsets in class coordinates)
  int local_stride = 0;
  if (local_bias) {
    if (args.local_radius < 0 || args.local_radius > (1 << 30)) return SWA_ERR_INVALID_ARG;
    int r_eff_max = 0;
    for (int h = 0; h < Hq; ++h) {
      const long long dh = dilation ? dilation[h] : 1;
      const long long reach = std::min((long long)window[h] * dh, (long long)d.seq_len - 1);
      if (args.local_radius < reach) return SWA_ERR_INVALID_ARG;
      const long long nc = (d.seq_len + dh - 1) / dh;
      r_eff_max = (int)std::max<long long>(r_eff_max, std::min<long long>(window[h], nc));
    }
    local_stride = (int)align_up(2 * (size_t)r_eff_max + 2 * kLocalPad + 4, 32);
    if (d.dtype == SWA_BF16 && local_stride > band_bias_copy(d.head_dim)) return SWA_ERR_UNSUPPORTED;
    // The band kernel keeps four copies of the row, shifted by 0..3 floats, local_stride
    // apart, and a 16-byte read takes copy (key offset & 3) at the offset rounded down
    // to 4.  Four consecutive rows (one quarter-warp step of that read) use the four
    // copies at one rounded offset: copies 8 floats past a multiple of 32 apart put
    // them on different shared-memory banks, where a multiple of 32 would stack them.
    if (local_stride + 8 <= band_bias_copy(d.head_dim)) local_stride += 8;
  }
  const bool bf16 = d.dtype == SWA_BF16;
  if (bf16 && num_global > 0 && (!ws.gq || !ws.gk || !ws.gv || !ws.part_o || !ws.part_lse))
    return SWA_ERR_INVALID_ARG;

  // ---------------------------------------------------------- parameters (on the stack)
  AttnParams p;
  memset(&p, 0, sizeof(p));
  const int n = d.seq_len, D = d.head_dim;
  p.B = d.batch;
  p.Hq = Hq;
  p.Hkv = d.num_kv_heads;
  p.n = n;
  p.D = D;
  p.G = Hq / d.num_kv_heads;
  p.g = num_global;
  p.gpad = num_global > 0 ? (int)align_up(num_global, kTile) : 0;
  p.S = d.num_side;
  p.side_block = d.num_side > 0 ? d.side_block : 1;
  p.nblk = d.num_side > 0 ? (n + d.side_block - 1) / d.side_block : 0;
  p.causal = causal;
  const float scale = d.scale > 0.f ? d.scale : 1.0f / sqrtf((float)D);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.valid_len = valid_len;
  p.global_idx = num_global > 0 ? global_idx : nullptr;
  p.bias = d.num_side > 0 ? bias : nullptr;
  p.local_bias = local_bias;
  p.local_radius = local_bias ? args.local_radius : 0;
  p.local_stride = local_stride;
  p.rand_blocks = rand_blocks;
  p.num_rand = rand_blocks ? args.num_rand : 0;
  p.out = out;
  p.lse = lse;
  p.err = ws.err;

  // residue classes: one per (distinct dilation value, residue)
  int nclass = 0;
  for (int h = 0; h < Hq; ++h) {
    const int dh = dilation ? dilation[h] : 1;
    p.window[h] = window[h];
    int base = -1;
    for (int c = 0; c < nclass; ++c)
      if (p.cls[c].d == dh && p.cls[c].c == 0) base = c;
    if (base < 0) {
      const int need = std::min(dh, n);
      if (nclass + need > kMaxClasses) return SWA_ERR_UNSUPPORTED;
      base = nclass;
      for (int c = 0; c < need; ++c) {
        p.cls[nclass].d = dh;
        p.cls[nclass].c = c;
        p.cls[nclass].n_c = (n - c + dh - 1) / dh;
        p.cls[nclass].nres = need;
        ++nclass;
      }
    }
    p.class_base[h] = base;
  }
  // Work units: two 128-row query tiles.  When query heads come in GQA pairs with
  // the same window and dilation (and no per-head side or local bias), a unit is the
  // same rows of two heads that share one KV head; otherwise it is two consecutive
  // row tiles of one head.  (Per-head bias rows are staged once per unit, so a
  // unit keeps one head when either bias is present.)
  {
    bool pair = (p.G % 2 == 0) && !(d.num_side > 0 && bias) && !local_bias;
    for (int h = 0; pair && h < Hq; h += 2)
      pair = window[h] == window[h + 1] && p.class_base[h] == p.class_base[h + 1];
    p.pair_heads = pair ? 1 : 0;
    for (int h = 0; h < Hq; ++h) {
      const int base = p.class_base[h];
      const int dh = p.cls[base].d;
      int units = 0;
      for (int c = 0; c < std::min(dh, n); ++c) {
        const int tiles = (p.cls[base + c].n_c + kTile - 1) / kTile;
        units += pair ? tiles : (tiles + 1) / 2;
      }
      p.tiles[h] = units;
    }
    // unit ids: (row unit, batch, head or head pair), heads fastest; heads with fewer
    // units than the largest skip the ids beyond theirs
    p.max_units = 0;
    for (int h = 0; h < Hq; ++h) p.max_units = std::max(p.max_units, p.tiles[h]);
  }
  if (num_global > 0) {
    p.dense_class = -1;
    for (int c = 0; c < nclass; ++c)
      if (p.cls[c].d == 1) p.dense_class = c;
    if (p.dense_class < 0) {
      if (nclass + 1 > kMaxClasses) return SWA_ERR_UNSUPPORTED;
      p.cls[nclass].d = 1;
      p.cls[nclass].c = 0;
      p.cls[nclass].n_c = n;
      p.cls[nclass].nres = 1;
      p.dense_class = nclass++;
    }
  }
  // tensor maps (bf16 tensor-core path)
  if (bf16) {
    const size_t row = (size_t)D * 2;
    bool ok = true;
    for (int c = 0; c < nclass && ok; ++c) {
      const int dd = p.cls[c].d, cc = p.cls[c].c, nc = p.cls[c].n_c;
      ok = ok && make_map(&p.mq[c], static_cast<const char*>(q) + cc * row, D, nc, (uint64_t)p.B * Hq,
                          dd * row, (uint64_t)n * row);
      ok = ok && make_map(&p.mk[c], static_cast<const char*>(k) + cc * row, D, nc,
                          (uint64_t)p.B * p.Hkv, dd * row, (uint64_t)n * row);
      ok = ok && make_map(&p.mv[c], static_cast<const char*>(v) + cc * row, D, nc,
                          (uint64_t)p.B * p.Hkv, dd * row, (uint64_t)n * row);
      ok = ok && make_map(&p.mo[c], static_cast<char*>(out) + cc * row, D, nc, (uint64_t)p.B * Hq,
                          dd * row, (uint64_t)n * row, true);
    }
    if (ok && num_global > 0) {
      p.part_o = ws.part_o;
      p.part_lse = ws.part_lse;
      ok = ok && make_map(&p.mgq, ws.gq, D, p.gpad, (uint64_t)p.B * Hq, row, (uint64_t)p.gpad * row);
      ok = ok && make_map(&p.mgk, ws.gk, D, p.gpad, (uint64_t)p.B * p.Hkv, row, (uint64_t)p.gpad * row);
      ok = ok && make_map(&p.mgv, ws.gv, D, p.gpad, (uint64_t)p.B * p.Hkv, row, (uint64_t)p.gpad * row);
    }
    if (ok && d.num_side > 0) {
      ok = ok && make_map(&p.msk, side_k, D, d.num_side, (uint64_t)p.B * p.Hkv, row,
                          (uint64_t)d.num_side * row);
      ok = ok && make_map(&p.msv, side_v, D, d.num_side, (uint64_t)p.B * p.Hkv, row,
                          (uint64_t)d.num_side * row);
    }
    if (!ok) return SWA_ERR_CUDA;
    // global-row split: at most one wave of CTAs over the key tiles (measured against
    // two waves and half a wave: fewer, longer units and fewer partials to merge)
    if (num_global > 0) {
      const int ntiles = (n + kTile - 1) / kTile;
      const int side_split = d.num_side > 0 ? 1 : 0;
      const long long units = (long long)p.B * Hq * (p.gpad / kTile);
      int want = (int)std::max(1LL, (long long)num_sms / units);
      want = std::min(want, std::min(ntiles, ws.nsplit_max - side_split));
      if (want < 1) return SWA_ERR_INVALID_ARG;
      const int tiles_per = (ntiles + want - 1) / want;
      p.split_keys = tiles_per * kTile;
      p.nsplit_keys = (n + p.split_keys - 1) / p.split_keys;
      p.nsplit = p.nsplit_keys + side_split;
    }
  }

  // ---------------------------------------------------------- launches
  int launches = 0;
  const bool debug = (d.flags & SWA_DEBUG_CHECKS) != 0;
  cudaError_t ce = cudaSuccess;
  if (debug && (num_global > 0 || rand_blocks)) {
    // Nothing that indexes with global_idx or the random blocks is enqueued until
    // the check has been read back.
    ce = launch_check_inputs(p, s);
    ++launches;
    *launches_out = launches;
    if (ce != cudaSuccess) return SWA_ERR_CUDA;
    const swa_status st = read_and_clear_error(ws.err, s);
    if (st != SWA_OK) return st;
  }
  if (build_side && bf16 && ws.agg_count && !local_bias && !rand_blocks) {
    // the band kernel builds the side keys / values in its prologue
    p.agg_k = k;
    p.agg_v = v;
    p.agg_sk = const_cast<void*>(side_k);
    p.agg_sv = const_cast<void*>(side_v);
    p.agg_count = ws.agg_count;
    if (cudaMemsetAsync(ws.agg_count, 0, sizeof(unsigned), s) != cudaSuccess) return SWA_ERR_CUDA;
  } else if (build_side) {
    ce = launch_side_aggregate_kv(k, v, const_cast<void*>(side_k), const_cast<void*>(side_v), d.batch,
                                  d.num_kv_heads, n, D, d.side_block, valid_len, bf16 ? 1 : 0, s);
    ++launches;
    if (ce != cudaSuccess) {
      *launches_out = launches;
      return SWA_ERR_CUDA;
    }
  }
  if (!bf16) {
    ce = launch_simt(p, q, k, v, side_k, side_v, 0, s);
    ++launches;
  } else {
    if (num_global > 0) {
      GatherSet gs = {{q, k, v}, {ws.gq, ws.gk, ws.gv}, {p.Hq, p.Hkv, p.Hkv}, {}, 3};
      ce = launch_gather_rows(gs, p.global_idx, p.B, p.n, p.g, p.gpad, p.D, 2, s);
      ++launches;
    }
    if (ce == cudaSuccess) {
      ce = launch_band_tc(p, num_sms, s);
      ++launches;
    }
    if (ce == cudaSuccess && num_global > 0) {
      ce = launch_global_rows_tc(p, num_sms, s);
      ++launches;
      if (ce == cudaSuccess) {
        ce = launch_merge_global_rows(p, 1, s);
        ++launches;
      }
    }
  }
  *launches_out = launches;
  if (ce != cudaSuccess) return SWA_ERR_CUDA;
  if (debug) return read_and_clear_error(ws.err, s);
  return SWA_OK;
}

}  // namespace swa
