// swa_kernels.h -- parameter blocks shared by the host runtime (swa_api.cu) and
// the device kernels.  Internal to the library; the public C ABI is
// include/swa.h.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace swa {

constexpr int kTile = 128;           // query rows per tile and keys per KV tile
constexpr int kMaxClasses = 16;      // distinct (dilation, residue) classes per forward
constexpr int kMaxHeads = 128;       // query heads per plan
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded waits: 2 s
constexpr int kBiasCopy = 2048;      // floats per staged bias copy (4 copies in shared memory)
constexpr int kLocalPad = 256;       // zero entries staged on each side of a local-bias row
constexpr int kMaxRand = 8;          // random key blocks per query block

// Bits of the device error word.
constexpr int kDevErrTimeout = 1;    // a bounded wait expired
constexpr int kDevErrCheck = 2;      // a device-side precondition check failed

// Residue class: positions c, c+d, c+2d, ... of one dilation value d.
struct ResidueClass {
  int d, c, n_c;                     // dilation, residue, rows in the class
  int nres;                          // classes of this dilation: min(d, n)
};

struct AttnParams {
  // Tensor maps (3-D: x = head_dim, y = row, z = batch*head plane).  Band maps are
  // per residue class: base + c*row, row stride d*row.
  CUtensorMap mq[kMaxClasses];
  CUtensorMap mk[kMaxClasses];
  CUtensorMap mv[kMaxClasses];
  CUtensorMap mo[kMaxClasses];       // out, same class views as mq (32-column store boxes)
  CUtensorMap mgq, mgk, mgv;         // gathered global rows [B*H, gpad, D]
  CUtensorMap msk, msv;              // side keys / values [B*Hkv, S, D]
  ResidueClass cls[kMaxClasses];

  int B, Hq, Hkv, n, D, G;           // G = Hq / Hkv
  int g, gpad, S, side_block, nblk, causal;
  int dense_class;                   // class id of (d = 1, c = 0): all rows, for global rows
  float scale_log2;                  // softmax scale * log2(e)

  const int32_t* valid_len;          // [B] or nullptr (= n)
  const int32_t* global_idx;         // [B, g] or nullptr
  const float* bias;                 // [Hq, S + nblk - 1] or nullptr
  const float* local_bias;           // [Hq, 2 * local_radius + 1] or nullptr (window keys)
  int local_radius;
  int local_stride;                  // floats per staged copy of a local-bias row (band kernel)
  const int32_t* rand_blocks;        // [B, Hq, nqb, num_rand] random key blocks, or nullptr
  int num_rand;                      // r (0: none); blocks are kTile keys, nqb = ceil(n / kTile)
  void* out;                         // [B, Hq, n, D], input dtype
  float* lse;                        // [B, Hq, n] or nullptr
  float* part_o;                     // global-row partials [nsplit, B*Hq, gpad, D]
  float* part_lse;                   // [nsplit, B*Hq, gpad]
  int nsplit_keys, split_keys, nsplit;  // global-row key splits (+1 for side keys)
  int pair_heads;                    // units pair heads 2m, 2m+1 (same rows) instead of row tiles
  int max_units;                     // largest tiles[h]
  int* err;                          // device error word
  // Fused Transient-Global prologue (MODE 0): every CTA first builds its share of
  // the side keys / values (block means of agg_k / agg_v into agg_sk / agg_sv, the
  // buffers msk / msv map), then counts itself done in *agg_count (zeroed before
  // the launch); side tiles are loaded once all gridDim.x CTAs are counted.  The
  // launch is cooperative, so every CTA is resident.  Null agg_count: side keys are inputs.
  const void* agg_k;
  const void* agg_v;
  void* agg_sk;
  void* agg_sv;
  unsigned* agg_count;

  int window[kMaxHeads];
  int class_base[kMaxHeads];         // class id of (dilation[h], c = 0)
  int tiles[kMaxHeads];              // work units of head h (of head pair h/2 when pairing)
};

// Launchers (each returns the launch's cudaError_t).
cudaError_t launch_band_tc(const AttnParams& p, int num_sms, cudaStream_t s);
cudaError_t launch_global_rows_tc(const AttnParams& p, int num_sms, cudaStream_t s);
cudaError_t launch_merge_global_rows(const AttnParams& p, int bf16_out, cudaStream_t s);
// Up to kMaxGather arrays gathered by one launch; `end` is filled by the launcher.
constexpr int kMaxGather = 4;
struct GatherSet {
  const void* src[kMaxGather];
  void* dst[kMaxGather];
  int heads[kMaxGather];
  size_t end[kMaxGather];
  int count;
};
// For every array of the set: dst[bh, e, :] = src[bh, gidx[b, e], :] for e < g, zeros up
// to gpad ([B*H, n, D] -> [B*H, gpad, D]); one launch for all of them.
cudaError_t launch_gather_rows(const GatherSet& set, const int32_t* gidx, int B, int n, int g, int gpad, int D,
                               int elem_bytes, cudaStream_t s);
cudaError_t launch_simt(const AttnParams& p, const void* q, const void* k, const void* v,
                        const void* side_k, const void* side_v, int bf16, cudaStream_t s);
// Debug check of the index inputs: global_idx rows strictly increasing inside
// [0, valid_len), random key blocks inside [0, ceil(n / 128)); sets kDevErrCheck.
cudaError_t launch_check_inputs(const AttnParams& p, cudaStream_t s);
cudaError_t launch_wait_probe(int* err, uint64_t limit_ns, cudaStream_t s);
cudaError_t launch_exp2_poly(const float* x, float* y, int n, cudaStream_t s);
cudaError_t launch_side_aggregate(const void* x, void* out, int B, int H, int n, int D, int kb,
                                  const int32_t* valid_len, int bf16, cudaStream_t s);
// Side keys and values (block means of k and v, as launch_side_aggregate) in one
// launch; D must be a multiple of 8 (bf16) or 4 (fp32), buffers 16-byte aligned.
cudaError_t launch_side_aggregate_kv(const void* k, const void* v, void* sk, void* sv, int B, int H,
                                     int n, int D, int kb, const int32_t* valid_len, int bf16,
                                     cudaStream_t s);
size_t band_tc_smem_bytes(int D);
int band_bias_copy(int D);           // floats per staged bias copy of the band kernel

}  // namespace swa
