// swa_api.cu -- host runtime behind the C ABI of include/swa.h: plan creation
// and workspace, argument validation, residue-class and TMA tensor-map set-up,
// and the launch sequence of one forward pass.
//
// Launch sequence of swa_forward (all on the caller's stream, no host sync):
//   bf16:  [debug: check global_idx] -> [g > 0: gather global q/k/v rows]
//          -> band kernel (window + global columns + side keys, every query row)
//          -> [g > 0: global-row kernel (split over keys) -> logsumexp merge that
//             overwrites the global query rows]
//   fp32:  [debug check] -> CUDA-core kernel (all rows, global rows included)
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <new>
#include <vector>

#include "../../include/swa.h"
#include "swa_kernels.h"
#include "bwd_kernels.h"

using swa::AttnParams;
using swa::kMaxClasses;
using swa::kMaxHeads;
using swa::kTile;

struct swa_plan_s {
  swa_plan_desc desc;
  int device;
  int gpad;            // global slots rounded up to a tile
  int nsplit_max;      // global-row splits the workspace holds
  char* ws;
  size_t ws_bytes;
  int* err;            // device error word
  void* gq;
  void* gk;
  void* gv;
  float* part_o;
  float* part_lse;
  float* delta;        // backward: rowsum(dout * out) [B, Hq, n]
  int last_launches;
  int num_sms;         // persistent grid size
};

namespace {

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_bytes(swa_dtype t) { return t == SWA_FP32 ? 4 : 2; }

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

// 3-D bf16 map: x = D, y = rows (box 128), z = planes (box 1).  Loads use a box
// of 64 columns with the 128-byte swizzle (the tcgen05 operand layout); output
// stores use a box of 32 columns with the 64-byte swizzle (the staging layout).
bool make_map(CUtensorMap* m, const void* base, int D, uint64_t rows, uint64_t planes,
              uint64_t row_stride_bytes, uint64_t plane_stride_bytes, bool store_box = false,
              int box_rows = kTile) {
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

swa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SWA_OK : SWA_ERR_CUDA; }

}  // namespace

extern "C" {

const char* swa_status_string(swa_status s) {
  switch (s) {
    case SWA_OK: return "SWA_OK";
    case SWA_ERR_INVALID_ARG: return "SWA_ERR_INVALID_ARG";
    case SWA_ERR_UNSUPPORTED: return "SWA_ERR_UNSUPPORTED";
    case SWA_ERR_CUDA: return "SWA_ERR_CUDA";
    case SWA_ERR_OOM: return "SWA_ERR_OOM";
    case SWA_ERR_TIMEOUT: return "SWA_ERR_TIMEOUT";
    case SWA_ERR_DEVICE_CHECK: return "SWA_ERR_DEVICE_CHECK";
  }
  return "SWA_ERR_UNKNOWN";
}

swa_status swa_plan_create(swa_plan_t* out_plan, const swa_plan_desc* d) {
  if (!out_plan || !d) return SWA_ERR_INVALID_ARG;
  *out_plan = nullptr;
  if (d->batch < 1 || d->seq_len < 1 || d->num_q_heads < 1 || d->num_kv_heads < 1 ||
      d->num_q_heads % d->num_kv_heads != 0 || d->max_global < 0 || d->num_side < 0 ||
      d->head_dim < 1 || (d->dtype != SWA_BF16 && d->dtype != SWA_FP32) || d->scale < 0.f ||
      !(d->scale == d->scale) || (d->num_side > 0 && d->side_block < 1) ||
      d->max_global > d->seq_len || (d->flags & ~SWA_DEBUG_CHECKS))
    return SWA_ERR_INVALID_ARG;
  if (d->head_dim != 64 && d->head_dim != 128) return SWA_ERR_UNSUPPORTED;
  if (d->num_q_heads > kMaxHeads) return SWA_ERR_UNSUPPORTED;
  if ((long long)d->batch * d->num_q_heads > 65535LL * 65535LL) return SWA_ERR_UNSUPPORTED;

  swa_plan_s* p = new (std::nothrow) swa_plan_s();
  if (!p) return SWA_ERR_OOM;
  p->desc = *d;
  if (cudaGetDevice(&p->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&p->num_sms, cudaDevAttrMultiProcessorCount, p->device) != cudaSuccess) {
    delete p;
    return SWA_ERR_CUDA;
  }
  const size_t es = elem_bytes(d->dtype);
  const size_t B = d->batch, Hq = d->num_q_heads, Hkv = d->num_kv_heads, D = d->head_dim;
  p->gpad = d->max_global > 0 ? (int)align_up(d->max_global, kTile) : 0;
  const int ntiles = (d->seq_len + kTile - 1) / kTile;
  p->nsplit_max = std::min(ntiles, 64) + 1;
  size_t off = 256;  // error word
  size_t o_gq = 0, o_gk = 0, o_gv = 0, o_po = 0, o_pl = 0;
  if (p->gpad > 0 && d->dtype == SWA_BF16) {
    o_gq = off; off = align_up(off + B * Hq * p->gpad * D * es, 256);
    o_gk = off; off = align_up(off + B * Hkv * p->gpad * D * es, 256);
    o_gv = off; off = align_up(off + B * Hkv * p->gpad * D * es, 256);
    o_po = off; off = align_up(off + (size_t)p->nsplit_max * B * Hq * p->gpad * D * 4, 256);
    o_pl = off; off = align_up(off + (size_t)p->nsplit_max * B * Hq * p->gpad * 4, 256);
  }
  size_t o_delta = 0;
  if (d->dtype == SWA_BF16) {
    o_delta = off;
    off = align_up(off + B * Hq * (size_t)d->seq_len * 4, 256);
  }
  p->ws_bytes = off;
  if (cudaMalloc(&p->ws, p->ws_bytes) != cudaSuccess) {
    cudaGetLastError();
    delete p;
    return SWA_ERR_OOM;
  }
  if (cudaMemset(p->ws, 0, 256) != cudaSuccess) {
    cudaFree(p->ws);
    delete p;
    return SWA_ERR_CUDA;
  }
  p->err = reinterpret_cast<int*>(p->ws);
  if (o_delta) p->delta = reinterpret_cast<float*>(p->ws + o_delta);
  if (o_gq) {
    p->gq = p->ws + o_gq;
    p->gk = p->ws + o_gk;
    p->gv = p->ws + o_gv;
    p->part_o = reinterpret_cast<float*>(p->ws + o_po);
    p->part_lse = reinterpret_cast<float*>(p->ws + o_pl);
  }
  *out_plan = p;
  return SWA_OK;
}

swa_status swa_plan_destroy(swa_plan_t p) {
  if (!p) return SWA_OK;
  int cur = -1;
  cudaGetDevice(&cur);
  if (cur != p->device) cudaSetDevice(p->device);
  cudaError_t e = cudaFree(p->ws);
  if (cur != p->device && cur >= 0) cudaSetDevice(cur);
  delete p;
  return e == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}

size_t swa_plan_workspace_bytes(swa_plan_t p) { return p ? p->ws_bytes : 0; }

int swa_plan_last_launches(swa_plan_t p) { return p ? p->last_launches : 0; }

swa_status swa_plan_check(swa_plan_t p, void* stream) {
  if (!p) return SWA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return SWA_ERR_CUDA;
  int h = 0;
  if (cudaMemcpy(&h, p->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SWA_ERR_CUDA;
  if (h) {
    if (cudaMemset(p->err, 0, sizeof(int)) != cudaSuccess) return SWA_ERR_CUDA;
  }
  if (h & swa::kDevErrTimeout) return SWA_ERR_TIMEOUT;
  if (h & swa::kDevErrCheck) return SWA_ERR_DEVICE_CHECK;
  return SWA_OK;
}

swa_status swa_forward(swa_plan_t plan, const void* q, const void* k, const void* v,
                       const int32_t* global_idx, int num_global, const void* side_k,
                       const void* side_v, const float* bias, const int32_t* window,
                       const int32_t* dilation, int causal, const int32_t* valid_len, void* out,
                       float* lse, void* stream) {
  swa_forward_args a;
  memset(&a, 0, sizeof(a));
  a.q = q;
  a.k = k;
  a.v = v;
  a.global_idx = global_idx;
  a.num_global = num_global;
  a.side_k = side_k;
  a.side_v = side_v;
  a.bias = bias;
  a.window = window;
  a.dilation = dilation;
  a.causal = causal;
  a.valid_len = valid_len;
  a.out = out;
  a.lse = lse;
  return swa_forward_ex(plan, &a, stream);
}

swa_status swa_forward_ex(swa_plan_t plan, const swa_forward_args* args, void* stream) {
  if (!plan || !args) return SWA_ERR_INVALID_ARG;
  const void *q = args->q, *k = args->k, *v = args->v;
  const int32_t* global_idx = args->global_idx;
  const int num_global = args->num_global;
  const void *side_k = args->side_k, *side_v = args->side_v;
  const float* bias = args->bias;
  const int32_t *window = args->window, *dilation = args->dilation;
  const int causal = args->causal;
  const int32_t* valid_len = args->valid_len;
  void* out = args->out;
  float* lse = args->lse;
  const float* local_bias = args->local_bias;
  const int32_t* rand_blocks = args->num_rand > 0 ? args->rand_blocks : nullptr;
  const swa_plan_desc& d = plan->desc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  plan->last_launches = 0;
  // ---------------------------------------------------------- validation
  if (!q || !k || !v || !out || !window) return SWA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SWA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SWA_ERR_INVALID_ARG;
  if (num_global < 0 || num_global > d.max_global) return SWA_ERR_INVALID_ARG;
  if (num_global > 0 && !global_idx) return SWA_ERR_INVALID_ARG;
  if (d.num_side > 0) {
    if (!side_k || !side_v) return SWA_ERR_INVALID_ARG;
    if (!aligned16(side_k) || !aligned16(side_v)) return SWA_ERR_INVALID_ARG;
  }
  if ((lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) ||
      (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)) ||
      (local_bias && (reinterpret_cast<uintptr_t>(local_bias) & 3u)) ||
      (rand_blocks && (reinterpret_cast<uintptr_t>(rand_blocks) & 3u)))
    return SWA_ERR_INVALID_ARG;
  if (args->num_rand < 0 || args->num_rand > swa::kMaxRand) return SWA_ERR_INVALID_ARG;
  if (args->num_rand > 0 && !rand_blocks) return SWA_ERR_INVALID_ARG;
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
    if (args->local_radius < 0 || args->local_radius > (1 << 30)) return SWA_ERR_INVALID_ARG;
    int r_eff_max = 0;
    for (int h = 0; h < Hq; ++h) {
      const long long dh = dilation ? dilation[h] : 1;
      const long long reach = std::min((long long)window[h] * dh, (long long)d.seq_len - 1);
      if (args->local_radius < reach) return SWA_ERR_INVALID_ARG;
      const long long nc = (d.seq_len + dh - 1) / dh;
      r_eff_max = (int)std::max<long long>(r_eff_max, std::min<long long>(window[h], nc));
    }
    local_stride = (int)align_up(2 * (size_t)r_eff_max + 2 * swa::kLocalPad + 4, 32);
    if (d.dtype == SWA_BF16 && local_stride > swa::kBiasCopy) return SWA_ERR_UNSUPPORTED;
  }

  // ---------------------------------------------------------- parameters
  AttnParams* pp = new (std::nothrow) AttnParams;
  if (!pp) return SWA_ERR_OOM;
  AttnParams& p = *pp;
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
  p.local_radius = local_bias ? args->local_radius : 0;
  p.local_stride = local_stride;
  p.rand_blocks = rand_blocks;
  p.num_rand = rand_blocks ? args->num_rand : 0;
  p.out = out;
  p.lse = lse;
  p.err = plan->err;

  // residue classes: one per (distinct dilation value, residue)
  int nclass = 0;
  int max_tiles = 0;
  swa_status st = SWA_OK;
  for (int h = 0; h < Hq && st == SWA_OK; ++h) {
    const int dh = dilation ? dilation[h] : 1;
    p.window[h] = window[h];
    int base = -1;
    for (int c = 0; c < nclass; ++c)
      if (p.cls[c].d == dh && p.cls[c].c == 0) base = c;
    if (base < 0) {
      const int need = std::min(dh, n);
      if (nclass + need > kMaxClasses) { st = SWA_ERR_UNSUPPORTED; break; }
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
  // the same window and dilation (and no per-head side bias), a unit is the same
  // rows of two heads that share one KV head; otherwise it is two consecutive
  // row tiles of one head.  (Per-head side or local bias rows are staged once per
  // unit, so a unit keeps one head when either is present.)
  if (st == SWA_OK) {
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
      max_tiles = std::max(max_tiles, units);
    }
  }
  if (st == SWA_OK && num_global > 0) {
    p.dense_class = -1;
    for (int c = 0; c < nclass; ++c)
      if (p.cls[c].d == 1) p.dense_class = c;
    if (p.dense_class < 0) {
      if (nclass + 1 > kMaxClasses) st = SWA_ERR_UNSUPPORTED;
      else {
        p.cls[nclass].d = 1;
        p.cls[nclass].c = 0;
        p.cls[nclass].n_c = n;
        p.cls[nclass].nres = 1;
        p.dense_class = nclass++;
      }
    }
  }
  if (st != SWA_OK) {
    delete pp;
    return st;
  }

  int launches = 0;
  cudaError_t ce = cudaSuccess;
  if ((d.flags & SWA_DEBUG_CHECKS) && num_global > 0) {
    ce = swa::launch_check_globals(p, s);
    ++launches;
  }

  if (d.dtype == SWA_FP32) {
    if (ce == cudaSuccess) {
      ce = swa::launch_simt(p, q, k, v, side_k, side_v, 0, s);
      ++launches;
    }
  } else {
    // ---------------------------------------------------------- tensor maps
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
      p.part_o = plan->part_o;
      p.part_lse = plan->part_lse;
      ok = ok && make_map(&p.mgq, plan->gq, D, p.gpad, (uint64_t)p.B * Hq, row, (uint64_t)p.gpad * row);
      ok = ok && make_map(&p.mgk, plan->gk, D, p.gpad, (uint64_t)p.B * p.Hkv, row, (uint64_t)p.gpad * row);
      ok = ok && make_map(&p.mgv, plan->gv, D, p.gpad, (uint64_t)p.B * p.Hkv, row, (uint64_t)p.gpad * row);
    }
    if (ok && d.num_side > 0) {
      ok = ok && make_map(&p.msk, side_k, D, d.num_side, (uint64_t)p.B * p.Hkv, row, (uint64_t)d.num_side * row);
      ok = ok && make_map(&p.msv, side_v, D, d.num_side, (uint64_t)p.B * p.Hkv, row, (uint64_t)d.num_side * row);
    }
    if (!ok) {
      delete pp;
      return SWA_ERR_CUDA;
    }
    // ---------------------------------------------------------- global-row split
    if (num_global > 0) {
      const int ntiles = (n + kTile - 1) / kTile;
      const long long units = (long long)p.B * Hq * (p.gpad / kTile);
      int want = (int)std::max(1LL, (2LL * 148 + units - 1) / units);
      want = std::min(want, std::min(ntiles, plan->nsplit_max - 1));
      const int tiles_per = (ntiles + want - 1) / want;
      p.split_keys = tiles_per * kTile;
      p.nsplit_keys = (n + p.split_keys - 1) / p.split_keys;
      p.nsplit = p.nsplit_keys + (d.num_side > 0 ? 1 : 0);
      if (ce == cudaSuccess) {
        ce = swa::launch_gather_globals(p, q, k, v, plan->gq, plan->gk, plan->gv, 2, s);
        launches += 3;
      }
    }
    if (ce == cudaSuccess) {
      p.max_units = max_tiles;
      ce = swa::launch_band_tc(p, plan->num_sms, s);
      ++launches;
    }
    if (ce == cudaSuccess && num_global > 0) {
      ce = swa::launch_global_rows_tc(p, plan->num_sms, s);
      ++launches;
      if (ce == cudaSuccess) {
        ce = swa::launch_merge_global_rows(p, 1, s);
        ++launches;
      }
    }
  }
  delete pp;
  plan->last_launches = launches;
  if (ce != cudaSuccess) return SWA_ERR_CUDA;
  if (d.flags & SWA_DEBUG_CHECKS) return swa_plan_check(plan, stream);
  return SWA_OK;
}

swa_status swa_backward(swa_plan_t plan, const swa_backward_args* a, void* stream) {
  if (!plan || !a) return SWA_ERR_INVALID_ARG;
  const swa_plan_desc& d = plan->desc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  plan->last_launches = 0;
  if (!a->q || !a->k || !a->v || !a->out || !a->lse || !a->dout || !a->window || !a->dq || !a->dk ||
      !a->dv)
    return SWA_ERR_INVALID_ARG;
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->out) ||
      !aligned16(a->dout) || !aligned16(a->dq) || !aligned16(a->dk) || !aligned16(a->dv) ||
      (reinterpret_cast<uintptr_t>(a->lse) & 3u))
    return SWA_ERR_INVALID_ARG;
  if (a->causal != 0 && a->causal != 1) return SWA_ERR_INVALID_ARG;
  const int Hq = d.num_q_heads, n = d.seq_len, D = d.head_dim;
  for (int h = 0; h < Hq; ++h) {
    if (a->window[h] < 0) return SWA_ERR_INVALID_ARG;
    if (a->dilation && a->dilation[h] < 1) return SWA_ERR_INVALID_ARG;
    if ((long long)a->window[h] * (a->dilation ? a->dilation[h] : 1) > (1LL << 30)) return SWA_ERR_INVALID_ARG;
  }
  if (d.dtype != SWA_BF16 || d.num_side > 0 || !plan->delta) return SWA_ERR_UNSUPPORTED;
  const int G = Hq / d.num_kv_heads;
  for (int h = 0; h < Hq; ++h) {
    const int h0 = (h / G) * G;
    if (a->window[h] != a->window[h0] || (a->dilation && a->dilation[h] != a->dilation[h0]))
      return SWA_ERR_UNSUPPORTED;
  }

  swa::BwdParams* pp = new (std::nothrow) swa::BwdParams;
  if (!pp) return SWA_ERR_OOM;
  swa::BwdParams& p = *pp;
  memset(&p, 0, sizeof(p));
  p.B = d.batch;
  p.Hq = Hq;
  p.Hkv = d.num_kv_heads;
  p.n = n;
  p.D = D;
  p.G = G;
  p.causal = a->causal;
  p.scale = d.scale > 0.f ? d.scale : 1.0f / sqrtf((float)D);
  p.scale_log2 = p.scale * 1.4426950408889634f;
  p.valid_len = a->valid_len;
  p.out = a->out;
  p.dout = a->dout;
  p.lse = a->lse;
  p.delta = plan->delta;
  p.dq = a->dq;
  p.dk = a->dk;
  p.dv = a->dv;
  p.err = plan->err;
  // residue classes (as in the forward) and tiles per head
  int nclass = 0;
  swa_status st = SWA_OK;
  for (int h = 0; h < Hq && st == SWA_OK; ++h) {
    const int dh = a->dilation ? a->dilation[h] : 1;
    p.window[h] = a->window[h];
    int base = -1;
    for (int c = 0; c < nclass; ++c)
      if (p.cls[c].d == dh && p.cls[c].c == 0) base = c;
    if (base < 0) {
      const int need = std::min(dh, n);
      if (nclass + need > kMaxClasses) { st = SWA_ERR_UNSUPPORTED; break; }
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
    int tiles = 0;
    for (int c = 0; c < std::min(dh, n); ++c) tiles += (p.cls[base + c].n_c + kTile - 1) / kTile;
    p.qtiles[h] = tiles;
    p.ktiles[h / G] = tiles;
    p.max_qtiles = std::max(p.max_qtiles, tiles);
    p.max_ktiles = std::max(p.max_ktiles, tiles);
  }
  if (st != SWA_OK) {
    delete pp;
    return st;
  }
  const size_t row = (size_t)D * 2;
  bool ok = true;
  for (int c = 0; c < nclass && ok; ++c) {
    const int dd = p.cls[c].d, cc = p.cls[c].c, nc = p.cls[c].n_c;
    ok = ok && make_map(&p.mq[c], static_cast<const char*>(a->q) + cc * row, D, nc, (uint64_t)p.B * Hq,
                        dd * row, (uint64_t)n * row);
    ok = ok && make_map(&p.mdo[c], static_cast<const char*>(a->dout) + cc * row, D, nc,
                        (uint64_t)p.B * Hq, dd * row, (uint64_t)n * row);
    ok = ok && make_map(&p.mk[c], static_cast<const char*>(a->k) + cc * row, D, nc,
                        (uint64_t)p.B * p.Hkv, dd * row, (uint64_t)n * row);
    ok = ok && make_map(&p.mv[c], static_cast<const char*>(a->v) + cc * row, D, nc,
                        (uint64_t)p.B * p.Hkv, dd * row, (uint64_t)n * row);
    // 64-row query / dout boxes for the key-stationary pass
    ok = ok && make_map(&p.mq64[c], static_cast<const char*>(a->q) + cc * row, D, nc, (uint64_t)p.B * Hq,
                        dd * row, (uint64_t)n * row, false, 64);
    ok = ok && make_map(&p.mdo64[c], static_cast<const char*>(a->dout) + cc * row, D, nc,
                        (uint64_t)p.B * Hq, dd * row, (uint64_t)n * row, false, 64);
  }
  if (!ok) {
    delete pp;
    return SWA_ERR_CUDA;
  }
  int launches = 0;
  cudaError_t ce = swa::launch_bwd_delta(p, s);
  ++launches;
  if (ce == cudaSuccess) {
    ce = swa::launch_bwd_dq(p, s);
    ++launches;
  }
  if (ce == cudaSuccess) {
    ce = swa::launch_bwd_dkv(p, s);
    ++launches;
  }
  delete pp;
  plan->last_launches = launches;
  if (ce != cudaSuccess) return SWA_ERR_CUDA;
  if (d.flags & SWA_DEBUG_CHECKS) return swa_plan_check(plan, stream);
  return SWA_OK;
}

swa_status swa_selftest_wait_timeout(swa_plan_t plan, uint64_t limit_ns, void* stream) {
  if (!plan || limit_ns == 0 || limit_ns > 5000000000ull) return SWA_ERR_INVALID_ARG;
  plan->last_launches = 1;
  return cuda_status(swa::launch_wait_probe(plan->err, limit_ns, static_cast<cudaStream_t>(stream)));
}

swa_status swa_side_aggregate(const void* x, void* out, int batch, int heads, int seq_len,
                              int head_dim, int block, const int32_t* valid_len, swa_dtype dtype,
                              void* stream) {
  if (!x || !out || batch < 1 || heads < 1 || head_dim < 1 || block < 1 || seq_len < block)
    return SWA_ERR_INVALID_ARG;
  if (dtype != SWA_BF16 && dtype != SWA_FP32) return SWA_ERR_INVALID_ARG;
  return cuda_status(swa::launch_side_aggregate(x, out, batch, heads, seq_len, head_dim, block, valid_len,
                                                dtype == SWA_BF16, static_cast<cudaStream_t>(stream)));
}

// T5 bidirectional bucket, 32 buckets and max distance 128: 16 per direction
// (+16 when delta > 0); |delta| < 8 exact; otherwise 8 + floor(2*log2(|delta|/8)),
// at most 15.  floor(2*log2(a/8)) >= m  <=>  a^2 >= 64 * 2^m, tested in integers.
int swa_relative_bucket(int delta) {
  int bucket = delta > 0 ? 16 : 0;
  const long long a = delta < 0 ? -(long long)delta : (long long)delta;
  if (a < 8) return bucket + (int)a;
  int step = 0;
  for (int m = 1; m <= 7; ++m)
    if (a * a >= (64LL << m)) step = m;
  return bucket + 8 + step;
}

swa_status swa_bucket_local_bias(int num_q_heads, int radius, const float* table, float* out) {
  if (num_q_heads < 1 || radius < 0 || radius > (1 << 28) || !table || !out) return SWA_ERR_INVALID_ARG;
  const size_t cols = 2 * (size_t)radius + 1;
  for (int h = 0; h < num_q_heads; ++h)
    for (size_t c = 0; c < cols; ++c)
      out[(size_t)h * cols + c] = table[h * 32 + swa_relative_bucket((int)c - radius)];
  return SWA_OK;
}

swa_status swa_expand_side_bias(int num_q_heads, int num_side, int nblk, const float* table,
                                float* out) {
  if (num_q_heads < 1 || num_side < 1 || nblk < 1 || !table || !out) return SWA_ERR_INVALID_ARG;
  const int cols = num_side + nblk - 1;
  for (int h = 0; h < num_q_heads; ++h)
    for (int c = 0; c < cols; ++c)
      out[(size_t)h * cols + c] = table[h * 32 + swa_relative_bucket(c - (nblk - 1))];
  return SWA_OK;
}

}  // extern "C"
