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
// the array.  Validation, set-up and the kernels launched are exactly those of
// swa_forward (swa_host.cu).
//
// Outside SWA_DEBUG_CHECKS mode nothing reads the error word back: this entry
// point never synchronises, and the next call clears the word.  An expired
// bounded wait is therefore only reported in debug mode, where every call
// synchronises and returns SWA_ERR_TIMEOUT or SWA_ERR_DEVICE_CHECK.
#include <cuda.h>
#include <cuda_runtime.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "../../include/swa.h"
#include "swa_host.h"
#include "swa_kernels.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[SWA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};

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
  if (!desc) return SWA_ERR_INVALID_ARG;
  const swa_plan_desc& d = *desc;
  const swa_status vs = swa::validate_desc(d);       // the checks of swa_plan_create
  if (vs != SWA_OK) return vs;
  if (num_global < 0 || num_global > d.max_global) return SWA_ERR_INVALID_ARG;

  // ---------------------------------------------------------- scratch layout
  // error word, then (bf16 with global tokens) the gathered global rows and as many
  // global-row splits as fit in the array
  swa::ForwardScratch ws;
  swa::GlobalLayout gl = {};
  int nsplit = 0;
  if (num_global > 0 && d.dtype == SWA_BF16) {
    const int gpad = (num_global + swa::kTile - 1) / swa::kTile * swa::kTile;
    const int side_split = d.num_side > 0 ? 1 : 0;
    nsplit = swa::max_global_splits(d);
    gl = swa::global_layout(d, gpad, nsplit, 256);
    while (nsplit > 1 + side_split && gl.end > (size_t)SWA_NOALLOC_SCRATCH_BYTES) {
      --nsplit;
      gl = swa::global_layout(d, gpad, nsplit, 256);
    }
    if (gl.end > (size_t)SWA_NOALLOC_SCRATCH_BYTES)
      return SWA_ERR_UNSUPPORTED;   // this problem needs more scratch than the static limit
  }
  void* scratch = nullptr;
  int num_sms = 0;
  swa_status st = scratch_for_current_device(&scratch, &num_sms);
  if (st != SWA_OK) return st;
  char* base = static_cast<char*>(scratch);
  ws.err = reinterpret_cast<int*>(base);
  if (nsplit > 0) {
    ws.gq = base + gl.gq;
    ws.gk = base + gl.gk;
    ws.gv = base + gl.gv;
    ws.part_o = reinterpret_cast<float*>(base + gl.po);
    ws.part_lse = reinterpret_cast<float*>(base + gl.pl);
    ws.nsplit_max = nsplit;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws.err, 0, sizeof(int), s) != cudaSuccess) return SWA_ERR_CUDA;

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
  int launches = 0;
  return swa::enqueue_forward(d, a, ws, num_sms, s, &launches);
}
