// swa_host.h -- host set-up shared by the entry points of include/swa.h: plan
// descriptor and forward-argument validation, residue classes and work units,
// TMA tensor maps, the global-row key split, and the launch sequence of one
// forward pass.  The plan-based forward (swa_api.cu) and the allocation-free
// forward (swa_noalloc.cu) differ only in where their scratch memory lives;
// everything else goes through enqueue_forward, so the two cannot drift apart.
// Internal to the library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/swa.h"
#include "swa_kernels.h"

namespace swa {

// Checks of a plan descriptor: SWA_ERR_INVALID_ARG for a value out of range,
// SWA_ERR_UNSUPPORTED for a valid shape the kernels do not implement.
swa_status validate_desc(const swa_plan_desc& d);

// Device scratch of one forward pass beyond its inputs and outputs.
struct ForwardScratch {
  int* err = nullptr;            // device error word (always present)
  void* gq = nullptr;            // gathered global q rows [B*Hq, gpad, D] (bf16 with global tokens)
  void* gk = nullptr;            // gathered global k / v rows [B*Hkv, gpad, D]
  void* gv = nullptr;
  float* part_o = nullptr;       // global-row partials [nsplit, B*Hq, gpad, D] fp32
  float* part_lse = nullptr;     // [nsplit, B*Hq, gpad]
  int nsplit_max = 0;            // splits part_o / part_lse hold (the side-key split included)
  void* side_k = nullptr;        // side keys / values built from k and v [B*Hkv, S, D] (plan
  void* side_v = nullptr;        // workspace; null where the caller must pass them)
  unsigned* agg_count = nullptr; // CTA counter of the band kernel's fused side-key prologue
};

// Bytes of one side key (or value) buffer a plan reserves for side_from_kv.
size_t side_buffer_bytes(const swa_plan_desc& d);

// Byte offsets of the global-token scratch for gpad global slots and nsplit
// splits, laid out from byte `base` (each piece 256-byte aligned).
struct GlobalLayout {
  size_t gq, gk, gv, po, pl, end;
};
GlobalLayout global_layout(const swa_plan_desc& d, int gpad, int nsplit, size_t base);

// Largest useful number of global-row splits: one per 128-key tile (at most 64)
// plus one for the side keys.
int max_global_splits(const swa_plan_desc& d);

// Synchronise `s`, read the device error word and clear it:
// SWA_ERR_TIMEOUT / SWA_ERR_DEVICE_CHECK / SWA_ERR_CUDA / SWA_OK.
swa_status read_and_clear_error(int* err, cudaStream_t s);

// 3-D bf16 TMA map: x = D, y = rows (box box_rows), z = planes (box 1).  Loads use
// 64-column boxes with the 128-byte swizzle (the tcgen05 operand layout); output
// stores use 32-column boxes with the 64-byte swizzle (the staging layout).
bool make_map(CUtensorMap* m, const void* base, int D, uint64_t rows, uint64_t planes,
              uint64_t row_stride_bytes, uint64_t plane_stride_bytes, bool store_box = false,
              int box_rows = kTile);

// Validate the arguments of one forward pass and enqueue it on `s`, with the
// scratch `ws` and a persistent grid of `num_sms` CTAs.  *launches receives the
// number of kernels enqueued.  In SWA_DEBUG_CHECKS mode the device check of
// global_idx (and of the random blocks) runs first and is read back before any
// kernel that indexes with them is enqueued; the call synchronises again at the
// end and reports the error word.
swa_status enqueue_forward(const swa_plan_desc& d, const swa_forward_args& a,
                           const ForwardScratch& ws, int num_sms, cudaStream_t s, int* launches);

}  // namespace swa
