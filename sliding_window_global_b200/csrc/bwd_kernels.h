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
  int num_sms;                       // grid of the persistent dq pass
  int max_ktiles;                    // largest ktiles[hk]
  // Terms beyond the band (all optional; see swa_backward_args).
  int extras;                        // any of the terms below is present
  int dense_class;                   // class of (d = 1, c = 0): every position, for non-band tiles
  const int32_t* global_idx;         // [B, g] or nullptr
  int g, gpad;
  CUtensorMap mgk, mgv;              // gathered global k / v rows [B*Hkv, gpad, D], 128-row boxes
  CUtensorMap mgq, mgdo;             // gathered global q / dout rows [B*Hq, gpad, D], 128-row boxes
  CUtensorMap mgq64, mgdo64;         // the same with 64-row boxes
  CUtensorMap msk, msv;              // side keys / values [B*Hkv, S, D]
  int S, side_block, nblk;
  const float* bias;                 // [Hq, S + nblk - 1] side bias or nullptr
  const float* local_bias;           // [Hq, 2 * local_radius + 1] or nullptr
  int local_radius;
  const int32_t* rand_blocks;        // [B, Hq, nqb, num_rand] or nullptr
  int num_rand;
  float* dsk;                        // [B, Hkv, S, D] fp32 side-key gradients
  float* dsv;
  int window[kMaxHeads];             // per query head (equal within a KV group)
  int class_base[kMaxHeads];         // per query head
  int qtiles[kMaxHeads];             // row tiles of query head h over its classes
  int ktiles[kMaxHeads];             // key tiles of KV head hk over its classes
};

cudaError_t launch_bwd_delta(const BwdParams& p, cudaStream_t s);
// dq of every query tile: band tiles, then (extras) global-column, side and random
// tiles; global query rows get only their window and side keys here.
cudaError_t launch_bwd_dq(const BwdParams& p, cudaStream_t s);
// dq of the global query rows over every key outside their window, added to dq.
cudaError_t launch_bwd_dq_global_rows(const BwdParams& p, cudaStream_t s);
// dk, dv of every key tile from the band's query tiles (and, with global tokens,
// from the global query rows whose window misses the key); overwrites dk, dv.
cudaError_t launch_bwd_dkv(const BwdParams& p, cudaStream_t s);
// dk, dv of the global keys from the rows whose window misses them, added to dk, dv.
cudaError_t launch_bwd_dkv_global_keys(const BwdParams& p, cudaStream_t s);
// dside_k, dside_v: every valid row attends every side key (overwrites).
cudaError_t launch_bwd_dkv_side(const BwdParams& p, cudaStream_t s);
// dk, dv of the random key blocks from the rows that drew them, added to dk, dv.
cudaError_t launch_bwd_dkv_random(const BwdParams& p, cudaStream_t s);

}  // namespace swa
