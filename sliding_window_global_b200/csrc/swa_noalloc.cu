// swa_noalloc.cu -- swa_forward_noalloc: the whole forward pass without a plan
// and without any allocation, for callers that cannot allocate memory at call
// time: code that runs under a strict memory budget or inside a host framework
// that hands out all device memory itself, real-time loops where an allocation
// (and the synchronisation a device allocation may imply) is not allowed, and
// plug-ins that may not create long-lived objects such as a plan.
//
// The only scratch memory the forward pass needs -- the device error word, the
// gathered rows of the global tokens and the split partial results of the
// global query rows -- lives in one file-scope __device__ array of
// SWA_NOALLOC_SCRATCH_BYTES.  Every device that loads this library holds that
// array until the process exits.  In host code the array's name only stands in
// for the symbol: its device address is obtained with cudaGetSymbolAddress, once
// per device, the first time this entry point runs on that device (with the
// device current), and that address is what the kernels receive.
//
// Every call shares the array, which keeps the previous call's contents: the
// error word is cleared by each call (on its stream) and everything else is
// completely rewritten before it is read.  Calls whose work overlaps on the GPU
// (different streams, or host threads, without ordering between them) race on
// the array.  The kernels launched are exactly those of swa_forward.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "../../include/swa.h"
#include "swa_kernels.h"

using swa::AttnParams;
using swa::kMaxClasses;
using swa::kMaxHeads;
using swa::kTile;

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[SWA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

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

// Same tensor-map shapes as the plan-based path: x = D, y = rows (box 128),
// z = planes; loads 64-column boxes with the 128-byte swizzle, output stores
// 32-column boxes with the 64-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int D, uint64_t rows, uint64_t planes,
              uint64_t row_stride_bytes, uint64_t plane_stride_bytes, bool store_box = false) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows == 0 || planes == 0) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, rows, planes};
  cuuint64_t strides[2] = {row_stride_bytes, plane_stride_bytes};
  cuuint32_t box[3] = {store_box ? 32u : 64u, (cuuint32_t)kTile, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE,
            store_box ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Device address of the scratch array (and SM count) on the current device,
// looked up on the first call per device.
swa_status scratch_for_current_device(void** addr, int* num_sms) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SWA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SWA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return SWA_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return SWA_ERR_CUDA;
    g_scratch_addr[dev] = ptr;
    g_num_sms[dev] = sms;
  }
  *addr = g_scratch_addr[dev];
  *num_sms = g_num_sms[dev];
  return SWA_OK;
}

}  // namespace

extern "C" swa_status swa_forward_noalloc(const swa_plan_desc* desc, const void* q, const void* k,
                                          const void* v, const int32_t* global_idx, int num_global,
                                          const void* side_k, const void* side_v, const float* bias,
                                          const int32_t* window, const int32_t* dilation, int causal,
                                          const int32_t* valid_len, void* out, float* lse,
                                          void* stream) {
  // ---------------------------------------------------------- descriptor
  if (!desc) return SWA_ERR_INVALID_ARG;
  const swa_plan_desc& d = *desc;
  if (d.batch < 1 || d.seq_len < 1 || d.num_q_heads < 1 || d.num_kv_heads < 1 ||
      d.num_q_heads % d.num_kv_heads != 0 || d.max_global < 0 || d.num_side < 0 || d.head_dim < 1 ||
      (d.dtype != SWA_BF16 && d.dtype != SWA_FP32) || d.scale < 0.f || !(d.scale == d.scale) ||
      (d.num_side > 0 && d.side_block < 1) || d.max_global > d.seq_len || (d.flags & ~SWA_DEBUG_CHECKS))
    return SWA_ERR_INVALID_ARG;
  if (d.head_dim != 64 && d.head_dim != 128) return SWA_ERR_UNSUPPORTED;
  if (d.num_q_heads > kMaxHeads) return SWA_ERR_UNSUPPORTED;
  // ---------------------------------------------------------- arguments
  if (!q || !k || !v || !out || !window) return SWA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SWA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SWA_ERR_INVALID_ARG;
  if (num_global < 0 || num_global > d.max_global) return SWA_ERR_INVALID_ARG;
  if (num_global > 0 && !global_idx) return SWA_ERR_INVALID_ARG;
  if (d.num_side > 0 && (!side_k || !side_v || !aligned16(side_k) || !aligned16(side_v)))
    return SWA_ERR_INVALID_ARG;
  if ((lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) || (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)))
    return SWA_ERR_INVALID_ARG;
  const int Hq = d.num_q_heads;
  for (int h = 0; h < Hq; ++h) {
    if (window[h] < 0) return SWA_ERR_INVALID_ARG;
    if (dilation && dilation[h] < 1) return SWA_ERR_INVALID_ARG;
    if ((long long)window[h] * (dilation ? dilation[h] : 1) > (1LL << 30)) return SWA_ERR_INVALID_ARG;
  }
  if (causal && num_global > 0) return SWA_ERR_UNSUPPORTED;

  // ---------------------------------------------------------- scratch layout
  const size_t B = d.batch, Hkv = d.num_kv_heads, D = d.head_dim;
  const int n = d.seq_len;
  const bool bf16 = d.dtype == SWA_BF16;
  const int gpad = num_global > 0 ? (int)align_up(num_global, kTile) : 0;
  const int ntiles = (n + kTile - 1) / kTile;
  size_t o_gq = 0, o_gk = 0, o_gv = 0, o_po = 0, o_pl = 0;
  int nsplit_max = 0;
  if (num_global > 0 && bf16) {
    const size_t gq_bytes = align_up(B * Hq * gpad * D * 2, 256);
    const size_t gkv_bytes = align_up(B * Hkv * gpad * D * 2, 256);
    const size_t per_split = align_up(B * Hq * gpad * D * 4, 256) + align_up(B * Hq * gpad * 4, 256);
    const size_t fixed = 256 + gq_bytes + 2 * gkv_bytes;
    const int side_split = d.num_side > 0 ? 1 : 0;
    nsplit_max = std::min(ntiles, 64) + side_split;
    while (nsplit_max > 1 + side_split &&
           fixed + (size_t)nsplit_max * per_split > (size_t)SWA_NOALLOC_SCRATCH_BYTES)
      --nsplit_max;
    if (fixed + (size_t)nsplit_max * per_split > (size_t)SWA_NOALLOC_SCRATCH_BYTES)
      return SWA_ERR_UNSUPPORTED;   // this problem needs more scratch than the static limit
    o_gq = 256;
    o_gk = o_gq + gq_bytes;
    o_gv = o_gk + gkv_bytes;
    o_po = o_gv + gkv_bytes;
    o_pl = o_po + (size_t)nsplit_max * align_up(B * Hq * gpad * D * 4, 256);
  }
  void* scratch = nullptr;
  int num_sms = 0;
  swa_status st = scratch_for_current_device(&scratch, &num_sms);
  if (st != SWA_OK) return st;
  char* ws = static_cast<char*>(scratch);
  int* err = reinterpret_cast<int*>(ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(err, 0, sizeof(int), s) != cudaSuccess) return SWA_ERR_CUDA;

  // ---------------------------------------------------------- parameters (on the stack)
  AttnParams p;
  memset(&p, 0, sizeof(p));
  const int Dh = d.head_dim;
  p.B = d.batch;
  p.Hq = Hq;
  p.Hkv = d.num_kv_heads;
  p.n = n;
  p.D = Dh;
  p.G = Hq / d.num_kv_heads;
  p.g = num_global;
  p.gpad = gpad;
  p.S = d.num_side;
  p.side_block = d.num_side > 0 ? d.side_block : 1;
  p.nblk = d.num_side > 0 ? (n + d.side_block - 1) / d.side_block : 0;
  p.causal = causal;
  const float scale = d.scale > 0.f ? d.scale : 1.0f / sqrtf((float)Dh);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.valid_len = valid_len;
  p.global_idx = num_global > 0 ? global_idx : nullptr;
  p.bias = d.num_side > 0 ? bias : nullptr;
  p.out = out;
  p.lse = lse;
  p.err = err;

  int nclass = 0;
  int max_units = 0;
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
  bool pair = (p.G % 2 == 0) && !(d.num_side > 0 && bias);
  for (int h = 0; pair && h < Hq; h += 2)
    pair = window[h] == window[h + 1] && p.class_base[h] == p.class_base[h + 1];
  p.pair_heads = pair ? 1 : 0;
  for (int h = 0; h < Hq; ++h) {
    const int base = p.class_base[h];
    int units = 0;
    for (int c = 0; c < std::min(p.cls[base].d, n); ++c) {
      const int tiles = (p.cls[base + c].n_c + kTile - 1) / kTile;
      units += pair ? tiles : (tiles + 1) / 2;
    }
    p.tiles[h] = units;
    max_units = std::max(max_units, units);
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

  // ---------------------------------------------------------- launches
  cudaError_t ce = cudaSuccess;
  if ((d.flags & SWA_DEBUG_CHECKS) && num_global > 0) ce = swa::launch_check_globals(p, s);
  if (!bf16) {
    if (ce == cudaSuccess) ce = swa::launch_simt(p, q, k, v, side_k, side_v, 0, s);
  } else {
    const size_t row = (size_t)Dh * 2;
    bool ok = true;
    for (int c = 0; c < nclass && ok; ++c) {
      const int dd = p.cls[c].d, cc = p.cls[c].c, nc = p.cls[c].n_c;
      ok = ok && make_map(&p.mq[c], static_cast<const char*>(q) + cc * row, Dh, nc, (uint64_t)p.B * Hq,
                          dd * row, (uint64_t)n * row);
      ok = ok && make_map(&p.mk[c], static_cast<const char*>(k) + cc * row, Dh, nc, (uint64_t)p.B * p.Hkv,
                          dd * row, (uint64_t)n * row);
      ok = ok && make_map(&p.mv[c], static_cast<const char*>(v) + cc * row, Dh, nc, (uint64_t)p.B * p.Hkv,
                          dd * row, (uint64_t)n * row);
      ok = ok && make_map(&p.mo[c], static_cast<char*>(out) + cc * row, Dh, nc, (uint64_t)p.B * Hq,
                          dd * row, (uint64_t)n * row, true);
    }
    void* gq = ws + o_gq;
    void* gk = ws + o_gk;
    void* gv = ws + o_gv;
    if (ok && num_global > 0) {
      p.part_o = reinterpret_cast<float*>(ws + o_po);
      p.part_lse = reinterpret_cast<float*>(ws + o_pl);
      ok = ok && make_map(&p.mgq, gq, Dh, gpad, (uint64_t)p.B * Hq, row, (uint64_t)gpad * row);
      ok = ok && make_map(&p.mgk, gk, Dh, gpad, (uint64_t)p.B * p.Hkv, row, (uint64_t)gpad * row);
      ok = ok && make_map(&p.mgv, gv, Dh, gpad, (uint64_t)p.B * p.Hkv, row, (uint64_t)gpad * row);
    }
    if (ok && d.num_side > 0) {
      ok = ok && make_map(&p.msk, side_k, Dh, d.num_side, (uint64_t)p.B * p.Hkv, row, (uint64_t)d.num_side * row);
      ok = ok && make_map(&p.msv, side_v, Dh, d.num_side, (uint64_t)p.B * p.Hkv, row, (uint64_t)d.num_side * row);
    }
    if (!ok) return SWA_ERR_CUDA;
    if (num_global > 0) {
      const long long units = (long long)p.B * Hq * (gpad / kTile);
      int want = (int)std::max(1LL, (2LL * num_sms + units - 1) / units);
      want = std::min(want, std::min(ntiles, nsplit_max - (d.num_side > 0 ? 1 : 0)));
      const int tiles_per = (ntiles + want - 1) / want;
      p.split_keys = tiles_per * kTile;
      p.nsplit_keys = (n + p.split_keys - 1) / p.split_keys;
      p.nsplit = p.nsplit_keys + (d.num_side > 0 ? 1 : 0);
      if (ce == cudaSuccess) ce = swa::launch_gather_globals(p, q, k, v, gq, gk, gv, 2, s);
    }
    p.max_units = max_units;
    if (ce == cudaSuccess) ce = swa::launch_band_tc(p, num_sms, s);
    if (ce == cudaSuccess && num_global > 0) {
      ce = swa::launch_global_rows_tc(p, num_sms, s);
      if (ce == cudaSuccess) ce = swa::launch_merge_global_rows(p, 1, s);
    }
  }
  if (ce != cudaSuccess) return SWA_ERR_CUDA;
  if (d.flags & SWA_DEBUG_CHECKS) {
    if (cudaStreamSynchronize(s) != cudaSuccess) return SWA_ERR_CUDA;
    int h = 0;
    if (cudaMemcpy(&h, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SWA_ERR_CUDA;
    if (h & swa::kDevErrTimeout) return SWA_ERR_TIMEOUT;
    if (h & swa::kDevErrCheck) return SWA_ERR_DEVICE_CHECK;
  }
  return SWA_OK;
}
