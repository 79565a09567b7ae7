// bwd_kernels.h -- parameter block and launchers of the backward pass (bwd_tc.cu).
// Internal to the library; the public C ABI is include/swa.h.
#pragma once

#include "swa_kernels.h"

namespace swa {

// Backward pass (band pattern: window, dilation, causal, GQA, padding).
struct BwdParams {
  CUtensorMap mq[kMaxClasses];       // class views of q, dout ([B*Hq] planes), k, v ([B*Hkv])
  CUtensorMap mdo[kMaxClasses];
  CUtensorMap mk[kMaxClasses];
  CUtensorMap mv[kMaxClasses];
  CUtensorMap mq64[kMaxClasses];     // q, dout with 64-row boxes (key-stationary pass)
  CUtensorMap mdo64[kMaxClasses];
  ResidueClass cls[kMaxClasses];
  int B, Hq, Hkv, n, D, G, causal;
  float scale, scale_log2;
  const int32_t* valid_len;          // [B] or nullptr
  const void* out;                   // [B, Hq, n, D] bf16 (forward output)
  const void* dout;                  // [B, Hq, n, D] bf16
  const float* lse;                  // [B, Hq, n] natural log
  float* delta;                      // [B, Hq, n] workspace: rowsum(dout * out)
  float* dq;                         // [B, Hq, n, D] fp32
  float* dk;                         // [B, Hkv, n, D] fp32
  float* dv;                         // [B, Hkv, n, D] fp32
  int* err;
  int max_qtiles;                    // largest qtiles[h]
  int max_ktiles;                    // largest ktiles[hk]
  int window[kMaxHeads];             // per query head (equal within a KV group)
  int class_base[kMaxHeads];         // per query head
  int qtiles[kMaxHeads];             // row tiles of query head h over its classes
  int ktiles[kMaxHeads];             // key tiles of KV head hk over its classes
};

cudaError_t launch_bwd_delta(const BwdParams& p, cudaStream_t s);
cudaError_t launch_bwd_dq(const BwdParams& p, cudaStream_t s);
cudaError_t launch_bwd_dkv(const BwdParams& p, cudaStream_t s);

}  // namespace swa
