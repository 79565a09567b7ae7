// swa_api.cu -- the plan-based entry points of include/swa.h: plan creation and
// workspace, swa_forward / swa_forward_ex (argument checks, parameter set-up and
// launches are shared with the allocation-free entry point in swa_host.cu), the
// backward pass, and the host helpers (bucket tables, side aggregation).
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
#include "swa_host.h"
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
  void* side_k;        // side keys / values built from k and v (side_from_kv)
  void* side_v;
  void* gdo;           // backward: gathered dout rows of the global tokens [B*Hq, gpad, D]
  int last_launches;
  int num_sms;         // persistent grid size
};

namespace {

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_bytes(swa_dtype t) { return t == SWA_FP32 ? 4 : 2; }

using swa::make_map;

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
  const swa_status vs = swa::validate_desc(*d);
  if (vs != SWA_OK) return vs;

  swa_plan_s* p = new (std::nothrow) swa_plan_s();
  if (!p) return SWA_ERR_OOM;
  p->desc = *d;
  if (cudaGetDevice(&p->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&p->num_sms, cudaDevAttrMultiProcessorCount, p->device) != cudaSuccess) {
    delete p;
    return SWA_ERR_CUDA;
  }
  const size_t es = elem_bytes(d->dtype);
  const size_t B = d->batch, Hq = d->num_q_heads;
  p->gpad = d->max_global > 0 ? (int)align_up(d->max_global, kTile) : 0;
  p->nsplit_max = swa::max_global_splits(*d);
  size_t off = 256;  // error word
  swa::GlobalLayout gl = {};
  if (p->gpad > 0 && d->dtype == SWA_BF16) {
    gl = swa::global_layout(*d, p->gpad, p->nsplit_max, off);
    off = gl.end;
  }
  size_t o_delta = 0;
  if (d->dtype == SWA_BF16) {
    o_delta = off;
    off = align_up(off + B * Hq * (size_t)d->seq_len * 4, 256);
  }
  size_t o_gdo = 0;
  if (p->gpad > 0 && d->dtype == SWA_BF16) {
    o_gdo = off;
    off = align_up(off + B * Hq * (size_t)p->gpad * d->head_dim * 2, 256);
  }
  size_t o_side = 0;
  const size_t side_bytes = swa::side_buffer_bytes(*d);
  if (side_bytes) {
    o_side = off;
    off += 2 * side_bytes;
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
  if (o_gdo) p->gdo = p->ws + o_gdo;
  if (o_side) {
    p->side_k = p->ws + o_side;
    p->side_v = p->ws + o_side + side_bytes;
  }
  if (gl.end) {
    p->gq = p->ws + gl.gq;
    p->gk = p->ws + gl.gk;
    p->gv = p->ws + gl.gv;
    p->part_o = reinterpret_cast<float*>(p->ws + gl.po);
    p->part_lse = reinterpret_cast<float*>(p->ws + gl.pl);
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
  return swa::read_and_clear_error(p->err, static_cast<cudaStream_t>(stream));
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
  swa::ForwardScratch ws;
  ws.err = plan->err;
  ws.gq = plan->gq;
  ws.gk = plan->gk;
  ws.gv = plan->gv;
  ws.part_o = plan->part_o;
  ws.part_lse = plan->part_lse;
  ws.nsplit_max = plan->nsplit_max;
  ws.side_k = plan->side_k;
  ws.side_v = plan->side_v;
  ws.agg_count = reinterpret_cast<unsigned*>(plan->ws + 64);   // inside the error-word block
  int launches = 0;
  const swa_status st = swa::enqueue_forward(plan->desc, *args, ws, plan->num_sms,
                                             static_cast<cudaStream_t>(stream), &launches);
  plan->last_launches = launches;
  return st;
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
  if (d.dtype != SWA_BF16 || !plan->delta) return SWA_ERR_UNSUPPORTED;
  // terms beyond the band (the forward's optional terms)
  const int num_global = a->num_global;
  const int32_t* rand_blocks = a->num_rand > 0 ? a->rand_blocks : nullptr;
  if (num_global < 0 || num_global > d.max_global || (num_global > 0 && !a->global_idx)) return SWA_ERR_INVALID_ARG;
  if (a->num_rand < 0 || a->num_rand > swa::kMaxRand || (a->num_rand > 0 && !rand_blocks)) return SWA_ERR_INVALID_ARG;
  if (d.num_side > 0 && (!a->side_k || !a->side_v || !a->dside_k || !a->dside_v || !aligned16(a->side_k) ||
                         !aligned16(a->side_v) || !aligned16(a->dside_k) || !aligned16(a->dside_v)))
    return SWA_ERR_INVALID_ARG;
  if ((a->bias && (reinterpret_cast<uintptr_t>(a->bias) & 3u)) ||
      (a->local_bias && (reinterpret_cast<uintptr_t>(a->local_bias) & 3u)))
    return SWA_ERR_INVALID_ARG;
  if (a->causal && num_global > 0) return SWA_ERR_UNSUPPORTED;
  if (rand_blocks) {
    if (a->causal) return SWA_ERR_UNSUPPORTED;
    for (int h = 0; h < Hq; ++h)
      if (a->dilation && a->dilation[h] != 1) return SWA_ERR_UNSUPPORTED;
  }
  if (a->local_bias) {
    if (a->local_radius < 0 || a->local_radius > (1 << 30)) return SWA_ERR_INVALID_ARG;
    for (int h = 0; h < Hq; ++h) {
      const long long reach = std::min((long long)a->window[h] * (a->dilation ? a->dilation[h] : 1),
                                       (long long)n - 1);
      if (a->local_radius < reach) return SWA_ERR_INVALID_ARG;
    }
  }
  if (num_global > 0 && (!plan->gq || !plan->gdo)) return SWA_ERR_UNSUPPORTED;
  const bool extras = num_global > 0 || d.num_side > 0 || a->local_bias || rand_blocks;
  const int G = Hq / d.num_kv_heads;
  for (int h = 0; h < Hq; ++h) {
    const int h0 = (h / G) * G;
    if (a->window[h] != a->window[h0] || (a->dilation && a->dilation[h] != a->dilation[h0]))
      return SWA_ERR_UNSUPPORTED;
  }

  swa::BwdParams p;   // on the stack: the call allocates nothing
  memset(&p, 0, sizeof(p));
  p.num_sms = plan->num_sms;
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
  p.extras = extras ? 1 : 0;
  p.global_idx = num_global > 0 ? a->global_idx : nullptr;
  p.g = num_global;
  p.gpad = num_global > 0 ? (int)align_up(num_global, kTile) : 0;
  p.S = d.num_side;
  p.side_block = d.num_side > 0 ? d.side_block : 1;
  p.nblk = d.num_side > 0 ? (n + d.side_block - 1) / d.side_block : 0;
  p.bias = d.num_side > 0 ? a->bias : nullptr;
  p.local_bias = a->local_bias;
  p.local_radius = a->local_bias ? a->local_radius : 0;
  p.rand_blocks = rand_blocks;
  p.num_rand = rand_blocks ? a->num_rand : 0;
  p.dsk = d.num_side > 0 ? a->dside_k : nullptr;
  p.dsv = d.num_side > 0 ? a->dside_v : nullptr;
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
  if (st != SWA_OK) return st;
  // the non-band jobs walk every position: the (d = 1, c = 0) class
  if (extras) {
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
  const size_t row = (size_t)D * 2;
  bool ok = true;
  if (num_global > 0) {
    const uint64_t gp = (uint64_t)p.gpad;
    ok = ok && make_map(&p.mgk, plan->gk, D, gp, (uint64_t)p.B * p.Hkv, row, gp * row);
    ok = ok && make_map(&p.mgv, plan->gv, D, gp, (uint64_t)p.B * p.Hkv, row, gp * row);
    ok = ok && make_map(&p.mgq, plan->gq, D, gp, (uint64_t)p.B * Hq, row, gp * row);
    ok = ok && make_map(&p.mgdo, plan->gdo, D, gp, (uint64_t)p.B * Hq, row, gp * row);
    ok = ok && make_map(&p.mgq64, plan->gq, D, gp, (uint64_t)p.B * Hq, row, gp * row, false, 64);
    ok = ok && make_map(&p.mgdo64, plan->gdo, D, gp, (uint64_t)p.B * Hq, row, gp * row, false, 64);
  }
  if (d.num_side > 0) {
    const uint64_t S = (uint64_t)d.num_side;
    ok = ok && make_map(&p.msk, a->side_k, D, S, (uint64_t)p.B * p.Hkv, row, S * row);
    ok = ok && make_map(&p.msv, a->side_v, D, S, (uint64_t)p.B * p.Hkv, row, S * row);
  }
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
  if (!ok) return SWA_ERR_CUDA;
  // Launch order: Delta; gathered global rows; dq (band + extra key tiles), then the
  // global rows' remaining keys added; dk/dv of the band (and the global rows'
  // remaining keys) written, then the global keys' and random blocks' remaining
  // rows added; the side keys' gradients.
  int launches = 0;
  cudaError_t ce = swa::launch_bwd_delta(p, s);
  ++launches;
  auto step = [&](cudaError_t (*fn)(const swa::BwdParams&, cudaStream_t)) {
    if (ce == cudaSuccess) {
      ce = fn(p, s);
      ++launches;
    }
  };
  if (num_global > 0 && ce == cudaSuccess) {
    const swa::GatherSet gs = {{a->q, a->dout, a->k, a->v}, {plan->gq, plan->gdo, plan->gk, plan->gv},
                               {Hq, Hq, p.Hkv, p.Hkv}, {}, 4};
    ce = swa::launch_gather_rows(gs, p.global_idx, p.B, n, num_global, p.gpad, D, 2, s);
    ++launches;
  }
  step(swa::launch_bwd_dq);
  if (num_global > 0) step(swa::launch_bwd_dq_global_rows);
  step(swa::launch_bwd_dkv);
  if (num_global > 0) step(swa::launch_bwd_dkv_global_keys);
  if (rand_blocks) step(swa::launch_bwd_dkv_random);
  if (d.num_side > 0) step(swa::launch_bwd_dkv_side);
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

swa_status swa_selftest_exp2_poly(const float* x, float* y, int n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return SWA_ERR_INVALID_ARG;
  return cuda_status(swa::launch_exp2_poly(x, y, n, static_cast<cudaStream_t>(stream)));
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
