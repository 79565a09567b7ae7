// aux_kernels.cu -- the non-tensor-core kernels of the library:
//   * gather of the global rows (q, k, v at the global positions) into dense
//     [B*H, gpad, D] buffers that the tensor-core kernel loads by TMA;
//   * logsumexp merge of the split global-row partials, overwriting the rows of
//     global queries (BigBird notes §3.2.3: a global token attends over the whole
//     sequence);
//   * the fp32 CUDA-core path (one warp per query row, online softmax) used for
//     fp32 inputs, where bf16 tensor-core products cannot meet fp32 accuracy;
//   * the Transient-Global block-mean aggregation that builds side keys/values
//     (LongT5 guide, Transient-Global: block summaries of k tokens);
//   * a device-side check of the global-index precondition.
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "side_mean.cuh"
#include "softmax_math.cuh"
#include "swa_kernels.h"

namespace swa {
namespace {

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// ------------------------------------------------------------------ gather
// dst[bh, e, :] = src[bh', global_idx[b, e], :] for e < g, zeros for g <= e < gpad.
// Every array of a GatherSet in one launch: the index range is the concatenation
// of the arrays' [B*H, gpad, row_vecs] ranges (job j ends at end[j]).
__global__ void gather_rows_kernel(const GatherSet gs, const int32_t* __restrict__ gidx, int n, int g, int gpad,
                                   int row_vecs, int B) {
  const size_t total = gs.end[gs.count - 1];
  for (size_t t = blockIdx.x * (size_t)blockDim.x + threadIdx.x; t < total;
       t += (size_t)gridDim.x * blockDim.x) {
    int jb = 0;
    while (jb + 1 < gs.count && t >= gs.end[jb]) ++jb;
    const size_t lt = t - (jb > 0 ? gs.end[jb - 1] : 0);
    const int x = (int)(lt % row_vecs);
    const size_t r = lt / row_vecs;
    const int e = (int)(r % gpad);
    const size_t bh = r / gpad;
    const int b = (int)(bh / gs.heads[jb]);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (e < g) {
      // a position outside the sequence (a broken precondition) gathers zeros
      // instead of reading out of bounds
      const int pos = gidx[(size_t)b * g + e];
      if (pos >= 0 && pos < n) v = static_cast<const uint4*>(gs.src[jb])[(bh * n + pos) * row_vecs + x];
    }
    static_cast<uint4*>(gs.dst[jb])[lt] = v;
  }
}

// ------------------------------------------------------------------ merge
// One warp per global row: o = sum_s w_s o_s / sum_s w_s, w_s = exp(lse_s - max).
template <typename T, int D>
__global__ void merge_global_rows_kernel(AttnParams p) {
  grid_dependency_wait();               // the partials of the global-row kernel before it
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int rows = p.B * p.Hq * p.g;
  if (warp >= rows) return;
  const int e = warp % p.g;
  const int bh = warp / p.g;
  const int b = bh / p.Hq;
  const size_t stride = (size_t)p.B * p.Hq * p.gpad;
  const size_t base = (size_t)bh * p.gpad + e;
  float m = -INFINITY;
  for (int s = 0; s < p.nsplit; ++s) m = fmaxf(m, p.part_lse[s * stride + base]);
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int x = 0; x < PER; ++x) acc[x] = 0.f;
  float wsum = 0.f;
  if (m > -INFINITY) {
    for (int s = 0; s < p.nsplit; ++s) {
      float ls = p.part_lse[s * stride + base];
      if (ls == -INFINITY) continue;
      float wgt = __expf(ls - m);
      wsum += wgt;
      const float* po = p.part_o + (s * stride + base) * D;
#pragma unroll
      for (int x = 0; x < PER; ++x) acc[x] += wgt * po[lane + 32 * x];
    }
  }
  const int pos = p.global_idx[(size_t)b * p.g + e];
  if (pos < 0 || pos >= p.n) return;      // broken precondition: never write out of bounds
  const size_t off = (size_t)bh * p.n + pos;
  T* o = static_cast<T*>(p.out) + off * D;
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
  for (int x = 0; x < PER; ++x) o[lane + 32 * x] = from_f<T>(acc[x] * inv);
  if (lane == 0 && p.lse) p.lse[off] = wsum > 0.f ? m + __logf(wsum) : -INFINITY;
}

// ------------------------------------------------------------------ fp32 CUDA-core path
// One warp per query row.  Keys are enumerated in the order: window keys, global
// keys (masked when already inside the window), side keys; a global query row
// instead walks every valid key, then the side keys.  32 keys per step: each lane
// scores one key, the warp updates the running max / sum with shuffles, and each
// lane accumulates D/32 output columns.
template <typename T, int D>
__global__ void simt_attn_kernel(AttnParams p, const T* __restrict__ q, const T* __restrict__ k,
                                 const T* __restrict__ v, const T* __restrict__ side_k,
                                 const T* __restrict__ side_v) {
  constexpr int PER = D / 32;
  __shared__ float sq[4][D];
  const int wib = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const size_t row = (size_t)blockIdx.x * 4 + wib;
  if (row >= (size_t)p.B * p.Hq * p.n) return;
  const int i = (int)(row % p.n);
  const int h = (int)((row / p.n) % p.Hq);
  const int b = (int)(row / ((size_t)p.n * p.Hq));
  const int hk = h / p.G;
  int V = p.valid_len ? p.valid_len[b] : p.n;
  if (V > p.n) V = p.n;
  T* orow = static_cast<T*>(p.out) + row * D;
  if (i >= V) {
#pragma unroll
    for (int x = 0; x < PER; ++x) orow[lane + 32 * x] = from_f<T>(0.f);
    if (lane == 0 && p.lse) p.lse[row] = -INFINITY;
    return;
  }
  const T* qi = q + row * D;
#pragma unroll
  for (int x = 0; x < PER; ++x) sq[wib][lane + 32 * x] = to_f<T>(qi[lane + 32 * x]);
  __syncwarp();
  const int r = p.window[h], d = p.cls[p.class_base[h]].d;
  const int32_t* gl = p.g ? p.global_idx + (size_t)b * p.g : nullptr;
  bool is_global = false;
  for (int t = 0; t < p.g; ++t) is_global |= (gl[t] == i);
  int t_lo = max(-r, -(i / d));
  int t_hi = p.causal ? 0 : min(r, (V - 1 - i) / d);
  const int nwin = is_global ? V : (t_hi - t_lo + 1);
  const int ngl = is_global ? 0 : p.g;
  // random key blocks of the row's query block (non-global rows)
  const int nqb = (p.n + kTile - 1) / kTile;
  const int32_t* rbp = (!is_global && p.rand_blocks)
                           ? p.rand_blocks + (((size_t)b * p.Hq + h) * nqb + i / kTile) * p.num_rand
                           : nullptr;
  const int nrnd = rbp ? p.num_rand * kTile : 0;
  const int total = nwin + ngl + p.S + nrnd;
  const T* kb = k + ((size_t)b * p.Hkv + hk) * p.n * D;
  const T* vb = v + ((size_t)b * p.Hkv + hk) * p.n * D;
  const T* skb = p.S ? side_k + ((size_t)b * p.Hkv + hk) * p.S * D : nullptr;
  const T* svb = p.S ? side_v + ((size_t)b * p.Hkv + hk) * p.S * D : nullptr;
  const float scale = p.scale_log2 * 0.6931471805599453f;  // natural-log scale
  const int qblk = p.S ? i / p.side_block : 0;
  float m = -INFINITY, l = 0.f;
  float acc[PER];
#pragma unroll
  for (int x = 0; x < PER; ++x) acc[x] = 0.f;
  for (int base = 0; base < total; base += 32) {
    const int idx = base + lane;
    float s = -INFINITY;
    const T* krow = nullptr;
    const T* vrow = nullptr;
    float bb = 0.f;
    if (idx < nwin) {
      int j = is_global ? idx : i + d * (t_lo + idx);
      krow = kb + (size_t)j * D;
      vrow = vb + (size_t)j * D;
      // local relative-position bias of window keys (offset j - i), non-global rows only
      if (!is_global && p.local_bias)
        bb = p.local_bias[(size_t)h * (2 * p.local_radius + 1) + p.local_radius + (j - i)];
    } else if (idx < nwin + ngl) {
      int j = gl[idx - nwin];
      int diff = i - j;
      bool inwin = (p.causal ? (diff >= 0 && diff <= r * d) : (abs(diff) <= r * d)) && (diff % d == 0);
      if (!inwin && j >= 0 && j < V) {
        krow = kb + (size_t)j * D;
        vrow = vb + (size_t)j * D;
      }
    } else if (idx < nwin + ngl + p.S) {
      int sg = idx - nwin - ngl;
      krow = skb + (size_t)sg * D;
      vrow = svb + (size_t)sg * D;
      if (p.bias) bb = p.bias[(size_t)h * (p.S + p.nblk - 1) + sg - qblk + p.nblk - 1];
    } else if (idx < total) {
      // key e of random block t: counted unless it is padded, in the window, global,
      // or in a block repeated earlier in the list
      const int rr = idx - nwin - ngl - p.S;
      const int t = rr / kTile;
      const int blk = rbp[t];
      const int j = blk * kTile + rr % kTile;
      bool take = blk >= 0 && blk < nqb && j < V;
      const int diff = i - j;
      const bool inwin = (p.causal ? (diff >= 0 && diff <= r * d) : (abs(diff) <= r * d)) && (diff % d == 0);
      take = take && !inwin;
      for (int u = 0; take && u < p.g; ++u) take = gl[u] != j;
      for (int t2 = 0; take && t2 < t; ++t2) take = rbp[t2] != blk;
      if (take) {
        krow = kb + (size_t)j * D;
        vrow = vb + (size_t)j * D;
      }
    }
    if (krow) {
      float dotv = 0.f;
#pragma unroll 8
      for (int x = 0; x < D; ++x) dotv = fmaf(sq[wib][x], to_f<T>(krow[x]), dotv);
      s = dotv * scale + bb;
    }
    float cmax = s;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
    const float m_new = fmaxf(m, cmax);
    if (m_new == -INFINITY) continue;
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
    const float pr = (s == -INFINITY) ? 0.f : expf(s - m_new);
    float psum = pr;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
    l = l * alpha + psum;
    m = m_new;
#pragma unroll
    for (int x = 0; x < PER; ++x) acc[x] *= alpha;
    for (int src = 0; src < 32; ++src) {
      const float ps = __shfl_sync(0xffffffffu, pr, src);
      const T* vr = reinterpret_cast<const T*>(
          __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(vrow), src));
      if (ps != 0.f) {
#pragma unroll
        for (int x = 0; x < PER; ++x) acc[x] = fmaf(ps, to_f<T>(vr[lane + 32 * x]), acc[x]);
      }
    }
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int x = 0; x < PER; ++x) orow[lane + 32 * x] = from_f<T>(acc[x] * inv);
  if (lane == 0 && p.lse) p.lse[row] = l > 0.f ? m + logf(l) : -INFINITY;
}

// ------------------------------------------------------------------ side aggregation
// out[b,h,s,:] = mean of x[b,h,j,:] over block s (j < valid_len); a trailing
// partial block joins the last full block; an empty block gives zeros.
template <typename T>
__global__ void side_aggregate_kernel(const T* __restrict__ x, T* __restrict__ out, int B, int H,
                                      int n, int D, int kb, const int32_t* __restrict__ valid_len) {
  const int S = n / kb;
  const size_t total = (size_t)B * H * S * D;
  for (size_t t = blockIdx.x * (size_t)blockDim.x + threadIdx.x; t < total;
       t += (size_t)gridDim.x * blockDim.x) {
    int col = (int)(t % D);
    size_t r = t / D;
    int s = (int)(r % S);
    size_t bh = r / S;
    int b = (int)(bh / H);
    int V = valid_len ? min(valid_len[b], n) : n;
    int lo = s * kb;
    int hi = (s == S - 1) ? n : lo + kb;
    hi = min(hi, V);
    float acc = 0.f;
    for (int j = lo; j < hi; ++j) acc += to_f<T>(x[(bh * n + j) * D + col]);
    int cnt = hi > lo ? hi - lo : 0;
    out[t] = from_f<T>(cnt ? acc / (float)cnt : 0.f);
  }
}

// Both side keys and side values in one launch (for the fp32 path of a forward
// handed raw K/V): the block means of side_aggregate_kernel, bit for bit, VEC
// consecutive columns per thread with 16-byte loads.  Threads [0, total) produce
// side keys, [total, 2 total) side values.
template <typename T>
__global__ void side_aggregate_kv_kernel(const T* __restrict__ k, const T* __restrict__ v,
                                         T* __restrict__ sk, T* __restrict__ sv, int B, int H, int n,
                                         int D, int kb, const int32_t* __restrict__ valid_len) {
  constexpr int VEC = 16 / sizeof(T);
  const int S = n / kb;
  const int groups = D / VEC;
  const size_t total = (size_t)B * H * S * groups;
  for (size_t t = blockIdx.x * (size_t)blockDim.x + threadIdx.x; t < 2 * total;
       t += (size_t)gridDim.x * blockDim.x) {
    const bool is_v = t >= total;
    const size_t u = is_v ? t - total : t;
    const int cg = (int)(u % groups);
    const size_t r = u / groups;
    const int s = (int)(r % S);
    const size_t bh = r / S;
    const int b = (int)(bh / H);
    const int V = valid_len ? min(valid_len[b], n) : n;
    side_mean_vec<T>(is_v ? v : k, is_v ? sv : sk, bh, s, cg, n, D, kb, V);
  }
}

// ------------------------------------------------------------------ precondition check
// global_idx rows must be strictly increasing and inside [0, valid_len); random
// key blocks must lie inside [0, nqb).  Threads [0, B*g) check global_idx, the
// next nrand_total threads the random blocks.
__global__ void check_inputs_kernel(const int32_t* __restrict__ gidx, int g, int B, int n,
                                    const int32_t* __restrict__ valid_len,
                                    const int32_t* __restrict__ rand_blocks, long long nrand_total,
                                    int nqb, int* err) {
  const long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  const long long ng = (long long)B * g;
  bool bad = false;
  if (t < ng) {
    const int b = (int)(t / g), e = (int)(t % g);
    const int V = valid_len ? min(valid_len[b], n) : n;
    const int pos = gidx[t];
    bad = pos < 0 || pos >= V || (e > 0 && gidx[t - 1] >= pos);
  } else if (t - ng < nrand_total) {
    const int blk = rand_blocks[t - ng];
    bad = blk < 0 || blk >= nqb;
  }
  if (bad) atomicOr(err, kDevErrCheck);
}

// ------------------------------------------------------------------ failure-path self test
// One thread waits on an mbarrier that nothing arrives at, with the bounded wait the
// attention kernels use; when the limit expires it reports a timeout in the error
// word, as those kernels do, and returns.
__global__ void wait_probe_kernel(int* err, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile int* a = &abort_flag;
    if (!mbar_wait_bounded(&bar, 0, a, limit_ns)) atomicOr(err, kDevErrTimeout);
  }
}

// ------------------------------------------------------------------ exp2 self test
// y = the band kernel's FMA-pipe 2^x (exp2_poly2), two elements per thread.
__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const long long i = 2 * (blockIdx.x * (long long)blockDim.x + threadIdx.x);
  if (i >= n) return;
  const bool two = i + 1 < n;
  float y0, y1;
  exp2_poly2(y0, y1, x[i], two ? x[i + 1] : 0.f);
  y[i] = y0;
  if (two) y[i + 1] = y1;
}

}  // namespace

cudaError_t launch_exp2_poly(const float* x, float* y, int n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const long long pairs = (n + 1LL) / 2;
  exp2_poly_kernel<<<(unsigned)((pairs + 255) / 256), 256, 0, s>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_wait_probe(int* err, uint64_t limit_ns, cudaStream_t s) {
  wait_probe_kernel<<<1, 32, 0, s>>>(err, limit_ns);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const GatherSet& set, const int32_t* gidx, int B, int n, int g, int gpad, int D,
                               int elem_bytes, cudaStream_t s) {
  if (set.count < 1 || set.count > kMaxGather) return cudaErrorInvalidValue;
  const int row_vecs = D * elem_bytes / 16;
  GatherSet gs = set;
  size_t total = 0;
  for (int j = 0; j < gs.count; ++j) {
    total += (size_t)B * gs.heads[j] * gpad * row_vecs;
    gs.end[j] = total;
  }
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const int blocks = (int)min((total + threads - 1) / threads, (size_t)4096);
  gather_rows_kernel<<<blocks, threads, 0, s>>>(gs, gidx, n, g, gpad, row_vecs, B);
  return cudaGetLastError();
}

cudaError_t launch_merge_global_rows(const AttnParams& p, int bf16_out, cudaStream_t s) {
  const int rows = p.B * p.Hq * p.g;
  const int threads = 256;
  const int blocks = (rows * 32 + threads - 1) / threads;
  // programmatic dependent launch behind the global-row kernel (the kernel waits)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(threads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (bf16_out)
    return p.D == 64 ? cudaLaunchKernelEx(&cfg, merge_global_rows_kernel<__nv_bfloat16, 64>, p)
                     : cudaLaunchKernelEx(&cfg, merge_global_rows_kernel<__nv_bfloat16, 128>, p);
  return p.D == 64 ? cudaLaunchKernelEx(&cfg, merge_global_rows_kernel<float, 64>, p)
                   : cudaLaunchKernelEx(&cfg, merge_global_rows_kernel<float, 128>, p);
}

cudaError_t launch_simt(const AttnParams& p, const void* q, const void* k, const void* v,
                        const void* side_k, const void* side_v, int bf16, cudaStream_t s) {
  const size_t rows = (size_t)p.B * p.Hq * p.n;
  const unsigned blocks = (unsigned)((rows + 3) / 4);
  if (bf16) {
    using T = __nv_bfloat16;
    if (p.D == 64)
      simt_attn_kernel<T, 64><<<blocks, 128, 0, s>>>(p, (const T*)q, (const T*)k, (const T*)v,
                                                      (const T*)side_k, (const T*)side_v);
    else
      simt_attn_kernel<T, 128><<<blocks, 128, 0, s>>>(p, (const T*)q, (const T*)k, (const T*)v,
                                                       (const T*)side_k, (const T*)side_v);
  } else {
    using T = float;
    if (p.D == 64)
      simt_attn_kernel<T, 64><<<blocks, 128, 0, s>>>(p, (const T*)q, (const T*)k, (const T*)v,
                                                      (const T*)side_k, (const T*)side_v);
    else
      simt_attn_kernel<T, 128><<<blocks, 128, 0, s>>>(p, (const T*)q, (const T*)k, (const T*)v,
                                                       (const T*)side_k, (const T*)side_v);
  }
  return cudaGetLastError();
}

cudaError_t launch_check_inputs(const AttnParams& p, cudaStream_t s) {
  const int nqb = (p.n + kTile - 1) / kTile;
  const long long nrand = p.rand_blocks ? (long long)p.B * p.Hq * nqb * p.num_rand : 0;
  const long long t = (long long)p.B * p.g + nrand;
  if (t == 0) return cudaSuccess;
  check_inputs_kernel<<<(unsigned)((t + 255) / 256), 256, 0, s>>>(p.global_idx, p.g, p.B, p.n, p.valid_len,
                                                                   p.rand_blocks, nrand, nqb, p.err);
  return cudaGetLastError();
}

cudaError_t launch_side_aggregate_kv(const void* k, const void* v, void* sk, void* sv, int B, int H,
                                     int n, int D, int kb, const int32_t* valid_len, int bf16,
                                     cudaStream_t s) {
  const int vec = bf16 ? 8 : 4;
  const size_t total = 2 * (size_t)B * H * (n / kb) * (D / vec);
  const int threads = 256;
  const int blocks = (int)min((total + threads - 1) / threads, (size_t)8192);
  if (bf16) {
    using T = __nv_bfloat16;
    side_aggregate_kv_kernel<T><<<blocks, threads, 0, s>>>((const T*)k, (const T*)v, (T*)sk, (T*)sv, B, H,
                                                              n, D, kb, valid_len);
  } else {
    side_aggregate_kv_kernel<float><<<blocks, threads, 0, s>>>((const float*)k, (const float*)v, (float*)sk,
                                                                  (float*)sv, B, H, n, D, kb, valid_len);
  }
  return cudaGetLastError();
}

cudaError_t launch_side_aggregate(const void* x, void* out, int B, int H, int n, int D, int kb,
                                  const int32_t* valid_len, int bf16, cudaStream_t s) {
  const size_t total = (size_t)B * H * (n / kb) * D;
  const int threads = 256;
  const int blocks = (int)min((total + threads - 1) / threads, (size_t)8192);
  if (bf16)
    side_aggregate_kernel<__nv_bfloat16><<<blocks, threads, 0, s>>>(
        (const __nv_bfloat16*)x, (__nv_bfloat16*)out, B, H, n, D, kb, valid_len);
  else
    side_aggregate_kernel<float><<<blocks, threads, 0, s>>>((const float*)x, (float*)out, B, H, n, D, kb,
                                                            valid_len);
  return cudaGetLastError();
}

}  // namespace swa
