/*
 * swa.h -- C ABI of the banded sparse self-attention library (libswa.so) for
 * NVIDIA B200 (sm_100a).
 *
 * What the library computes (forward pass, one call).  For every batch b, query
 * head h (KV head h / (Hq/Hkv)) and query position i < valid_len[b]:
 *   - the key set K(i) is the sliding window W(i) = { i + d*t : -r <= t <= r }
 *     (causal: -r <= t <= 0) clipped to [0, valid_len[b]), with r = window[h] and
 *     d = dilation[h] -- "精读笔记：Big Bird" §3.2.1 (query i attends i-w/2 .. i+w/2),
 *     the Longformer page §二 (dilated window: skip tokens inside the window), and
 *     SWAN-GPT §3.3(1) (fixed 512-key causal window in the SWA-RoPE layers);
 *   - united, as a set, with the global positions global_idx[b][:]; a global query
 *     instead attends every valid key (BigBird §3.2.3, internal/ITC global tokens;
 *     Longformer page §二 global attention);
 *   - plus every side key s in [0, S) of the LongT5 Transient-Global attention
 *     ("LongT5 长序列模型完全指南": Transient-Global block summaries as extra keys,
 *     with a global relative-position bias added to their scores);
 *   score = scale * <q_i, k_j>  (+ bias[h][s - floor(i / side_block) + nblk - 1] on
 *   side keys, nblk = ceil(seq_len / side_block)); o_i = softmax(scores) . V;
 *   lse_i = natural-log logsumexp of the scores.  Padded query rows
 *   (i >= valid_len[b]) give o = 0 and lse = -inf; padded keys are never attended.
 *
 * Layouts: every tensor is row-major and contiguous.
 *   q, out      [B, Hq,  n, D]      dtype of the plan (bf16 or fp32)
 *   k, v        [B, Hkv, n, D]
 *   side_k/v    [B, Hkv, S, D]
 *   bias        [Hq, S + nblk - 1]  fp32
 *   lse         [B, Hq, n]          fp32
 *   global_idx  [B, g]              int32, each row strictly increasing, < valid_len[b]
 *   valid_len   [B]                 int32 (trailing padding), or NULL for "no padding"
 *
 * Ownership: the caller owns every tensor.  The plan owns its workspace
 * (allocated by swa_plan_create, freed by swa_plan_destroy).  swa_forward neither
 * allocates nor synchronises (except in SWA_DEBUG_CHECKS mode) and never aborts
 * the process: every failure is a returned status.
 *
 * Threads and streams: one plan may be used by one stream at a time (its
 * workspace is reused by every forward).
 */
#ifndef SWA_H_
#define SWA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct swa_plan_s* swa_plan_t;

typedef enum {
  SWA_OK = 0,
  SWA_ERR_INVALID_ARG = 1,   /* a null/misaligned pointer, a bad size or value */
  SWA_ERR_UNSUPPORTED = 2,   /* valid request outside what the kernels implement */
  SWA_ERR_CUDA = 3,          /* a CUDA runtime/driver call or launch failed */
  SWA_ERR_OOM = 4,           /* workspace allocation failed */
  SWA_ERR_TIMEOUT = 5,       /* a bounded device-side wait expired (kernel returned early) */
  SWA_ERR_DEVICE_CHECK = 6   /* a device-side precondition check failed (debug mode) */
} swa_status;

typedef enum { SWA_BF16 = 0, SWA_FP32 = 1 } swa_dtype;

/* Plan flags. */
#define SWA_DEBUG_CHECKS 1u  /* check global_idx on the device and synchronise after
                                each forward, reporting device errors as a status */

typedef struct {
  int batch;           /* B >= 1 */
  int seq_len;         /* n >= 1 */
  int num_q_heads;     /* Hq >= 1, <= 128 */
  int num_kv_heads;    /* Hkv >= 1, Hq % Hkv == 0 */
  int head_dim;        /* D: 64 or 128 */
  swa_dtype dtype;     /* element type of q, k, v, side_k, side_v, out */
  int max_global;      /* largest g any forward will pass (0: no global tokens) */
  int num_side;        /* S >= 0 side keys per (batch, KV head) */
  int side_block;      /* k > 0 when num_side > 0: query block size of the side bias */
  float scale;         /* score scale; 0 selects 1/sqrt(head_dim) */
  unsigned flags;      /* SWA_DEBUG_CHECKS */
} swa_plan_desc;

/* Validate the descriptor and allocate the plan and its device workspace on the
 * current CUDA device.  Returns SWA_ERR_INVALID_ARG for a null argument or a
 * value out of range, SWA_ERR_UNSUPPORTED for head_dim not in {64, 128},
 * SWA_ERR_OOM when the workspace cannot be allocated. */
swa_status swa_plan_create(swa_plan_t* out_plan, const swa_plan_desc* desc);

/* One forward pass, enqueued on `stream` (a cudaStream_t; NULL = legacy default).
 *   q, k, v       device, required, 16-byte aligned
 *   global_idx    device [B, num_global] or NULL when num_global == 0;
 *                 0 <= num_global <= max_global
 *   side_k/v      device [B, Hkv, S, D], required when num_side > 0, else ignored
 *   bias          device [Hq, S + nblk - 1] fp32, or NULL (no bias)
 *   window        HOST [Hq] one-sided radius r >= 0 per query head
 *   dilation      HOST [Hq] d >= 1 per query head, or NULL (all 1)
 *   causal        0 or 1
 *   valid_len     device [B], or NULL (= seq_len)
 *   out           device [B, Hq, n, D], plan dtype, required
 *   lse           device [B, Hq, n] fp32, or NULL
 * Returns SWA_ERR_INVALID_ARG for a null required pointer, a pointer not 16-byte
 * aligned, window < 0, dilation < 1, num_global out of range; SWA_ERR_UNSUPPORTED
 * for causal together with num_global > 0, or more than 16 distinct
 * (dilation, residue) classes; SWA_ERR_CUDA when a launch fails.  In
 * SWA_DEBUG_CHECKS mode a device kernel first checks global_idx (and the random
 * blocks of swa_forward_ex); the call synchronises and reads the result back
 * before it enqueues anything that indexes with them, returning
 * SWA_ERR_DEVICE_CHECK with only that check launched; after the forward it
 * synchronises again and returns SWA_ERR_TIMEOUT if a bounded wait expired.
 * Outside debug mode the index preconditions are not checked; a position outside
 * [0, seq_len) still never makes a kernel read or write out of bounds (its
 * gathered row is zero and its global row is not written), but the results are
 * then undefined. */
swa_status swa_forward(swa_plan_t plan, const void* q, const void* k, const void* v,
                       const int32_t* global_idx, int num_global, const void* side_k,
                       const void* side_v, const float* bias, const int32_t* window,
                       const int32_t* dilation, int causal, const int32_t* valid_len, void* out,
                       float* lse, void* stream);

/* Arguments of swa_forward_ex: those of swa_forward, plus optional terms of the
 * score that swa_forward does not take.  Zero-initialise the struct (fields may
 * be appended in later versions; a zero field keeps its swa_forward meaning).
 *
 * local_bias: LongT5 local attention relative-position bias ("LongT5 长序列模型完全指南",
 *   相对位置编码 section: a bias bucketed on memory_position - query_position,
 *   computed once over the local window).  Device [Hq, 2*local_radius + 1] fp32,
 *   4-byte aligned, or NULL.  For a query i that is not a global token and a key
 *   j of its window W(i), local_bias[h][(j - i) + local_radius] is added to the
 *   score (natural-log units, like bias).  Global query rows, global keys outside
 *   W(i) and side keys get none; a global key inside W(i) is a window key.
 *   local_radius must be >= min(window[h] * dilation[h], seq_len - 1) for every
 *   head (else SWA_ERR_INVALID_ARG).  The bf16 kernels stage the bias rows of a
 *   work unit in shared memory, which limits min(window[h], ceil(seq_len /
 *   dilation[h])) to 766; larger windows with a local bias return
 *   SWA_ERR_UNSUPPORTED.  Use swa_bucket_local_bias to expand a 32-bucket table.
 *
 * rand_blocks, num_rand: BigBird random attention ("精读笔记：Big Bird" §3.2.2:
 *   every query also attends to r randomly chosen keys), in blocks of 128 keys.
 *   Device [B, Hq, ceil(seq_len / 128), num_rand] int32, 4-byte aligned: the
 *   rows of query block q = floor(i / 128) of head h add the keys of blocks
 *   rand_blocks[b][h][q][:] (keys 128*blk .. 128*blk + 127 below valid_len) to
 *   their key set, as a set: keys already in the window or global, and repeated
 *   blocks, count once.  Global query rows are unaffected (they attend every
 *   key).  The caller draws the blocks.  0 <= num_rand <= 8; block indices must
 *   lie in [0, ceil(seq_len / 128)) (checked in SWA_DEBUG_CHECKS mode; outside
 *   it an index outside attends nothing).  Random blocks need dilation 1 on every
 *   head and causal == 0 (else SWA_ERR_UNSUPPORTED).
 *
 * side_from_kv: 1 to have the forward build the Transient-Global side keys and
 *   values itself from k and v ("LongT5 长序列模型完全指南", Transient-Global: the
 *   tokens of each side_block-token block are summed and normalised into one
 *   global token; 源码级证据: padding tokens belong to no block, a trailing
 *   partial block joins the previous one) -- the block means that
 *   swa_side_aggregate computes, bit for bit, into the plan's workspace.  In a
 *   bf16 plan the band kernel builds them in a prologue (each CTA its share,
 *   launched cooperatively so that every CTA is resident; a CTA loads side tiles
 *   once all CTAs have counted themselves done, a wait bounded like the others),
 *   so the forward stays one launch; an fp32 plan runs one block-mean launch for
 *   k and v first.  side_k and side_v must then be NULL, and the plan's num_side
 *   must equal seq_len / side_block (else SWA_ERR_INVALID_ARG).  0 (the
 *   default): side_k / side_v are inputs. */
typedef struct {
  const void* q;
  const void* k;
  const void* v;
  const int32_t* global_idx;
  int num_global;
  const void* side_k;
  const void* side_v;
  const float* bias;
  const int32_t* window;       /* HOST */
  const int32_t* dilation;     /* HOST */
  int causal;
  const int32_t* valid_len;
  void* out;
  float* lse;
  const float* local_bias;     /* device [Hq, 2 * local_radius + 1] fp32, or NULL */
  int local_radius;
  const int32_t* rand_blocks;  /* device [B, Hq, ceil(n / 128), num_rand] int32, or NULL */
  int num_rand;
  int side_from_kv;            /* 1: build side keys / values from k and v (block means) */
} swa_forward_args;

/* swa_forward with the arguments in a struct (same statuses, same launches). */
swa_status swa_forward_ex(swa_plan_t plan, const swa_forward_args* args, void* stream);

/* Host helper: expand a per-head 32-bucket table [Hq][32] into the local-bias
 * table [Hq][2R + 1] that swa_forward_ex reads, column c holding the T5
 * bidirectional bucket of delta = c - R (memory position minus query position;
 * the bucket function of swa_relative_bucket).  Host pointers. */
swa_status swa_bucket_local_bias(int num_q_heads, int radius, const float* table, float* out);

/* ---------------------------------------------------------------------------
 * Backward pass: gradients of the forward's output with respect to q, k and v,
 * through the chain rule of each row's softmax (p = exp(s - lse), dp = dout . v,
 * ds = p (dp - rowsum(dout * out)), dq = scale ds k, dk = scale ds^T q,
 * dv = p^T dout) over the same key sets: the dilated / causal sliding window
 * ("精读笔记：Big Bird" §3.2.1, the Longformer page §二, SWAN-GPT §3.3(1)) with GQA
 * and padding, plus, when their fields are set, the other terms of the forward:
 * global rows and columns (BigBird §3.2.3), the Transient-Global side keys and
 * their bias (LongT5 guide, Transient-Global; gradients of the side keys and
 * values in dside_k / dside_v), the local relative-position bias (LongT5 guide,
 * 相对位置编码) and random blocks (BigBird §3.2.2).  The biases are inputs: no
 * gradient is formed for them.  The terms must be those the forward ran with
 * (its out and lse are read).  bf16 plans only (else SWA_ERR_UNSUPPORTED); the
 * query heads of one KV head must share window and dilation (else
 * SWA_ERR_UNSUPPORTED).  Gradients are written in fp32; dk and dv hold the sums
 * over the query heads of each KV head.  Every element of dq, dk, dv (and
 * dside_k, dside_v) is written (padded rows get 0).  The plan's workspace holds
 * rowsum(dout * out) and, with global tokens, the gathered global rows.
 * ------------------------------------------------------------------------- */
typedef struct {
  const void* q;               /* device [B, Hq, n, D] bf16, 16-byte aligned */
  const void* k;               /* device [B, Hkv, n, D] bf16 */
  const void* v;               /* device [B, Hkv, n, D] bf16 */
  const void* out;             /* device [B, Hq, n, D] bf16: the forward's output */
  const float* lse;            /* device [B, Hq, n] fp32: the forward's lse */
  const void* dout;            /* device [B, Hq, n, D] bf16: upstream gradient */
  const int32_t* window;       /* HOST [Hq] */
  const int32_t* dilation;     /* HOST [Hq] or NULL (all 1) */
  int causal;
  const int32_t* valid_len;    /* device [B] or NULL */
  float* dq;                   /* device [B, Hq, n, D] fp32 */
  float* dk;                   /* device [B, Hkv, n, D] fp32 */
  float* dv;                   /* device [B, Hkv, n, D] fp32 */
  /* Optional terms, as in swa_forward_ex (zero-initialise the struct; zero fields
   * keep the band-only meaning): */
  const int32_t* global_idx;   /* device [B, num_global] int32 or NULL */
  int num_global;              /* <= the plan's max_global */
  const void* side_k;          /* device [B, Hkv, S, D] bf16, required when the plan has side keys */
  const void* side_v;
  const float* bias;           /* device [Hq, S + nblk - 1] fp32 side bias, or NULL */
  const float* local_bias;     /* device [Hq, 2 * local_radius + 1] fp32, or NULL */
  int local_radius;
  const int32_t* rand_blocks;  /* device [B, Hq, ceil(n / 128), num_rand] int32, or NULL */
  int num_rand;
  float* dside_k;              /* device [B, Hkv, S, D] fp32, required when the plan has side keys */
  float* dside_v;
} swa_backward_args;

/* Three launches on `stream`: rowsum(dout * out), the query-stationary dq pass,
 * the key-stationary dk/dv pass.  Statuses as swa_forward. */
swa_status swa_backward(swa_plan_t plan, const swa_backward_args* args, void* stream);

/* Synchronise `stream` and read (then clear) the plan's device error word:
 * SWA_ERR_TIMEOUT if a bounded wait expired in any kernel since the last check,
 * SWA_ERR_DEVICE_CHECK if a precondition check failed, SWA_ERR_CUDA if the
 * stream reports an error, else SWA_OK. */
swa_status swa_plan_check(swa_plan_t plan, void* stream);

/* Release the workspace and the plan (NULL is accepted). */
swa_status swa_plan_destroy(swa_plan_t plan);

/* Bytes of device workspace the plan holds. */
size_t swa_plan_workspace_bytes(swa_plan_t plan);

/* Number of kernel launches the most recent swa_forward enqueued. */
int swa_plan_last_launches(swa_plan_t plan);

/* Self-test of the failure path (an addition of this library: the pages describe
 * nothing like it).  Enqueues one small kernel that waits, with the bounded wait
 * every kernel of the library uses, on a barrier that nothing signals; after
 * limit_ns (0 < limit_ns <= 5e9, else SWA_ERR_INVALID_ARG) the wait gives up and
 * sets the timeout bit of the plan's error word, as an expired wait in the
 * attention kernels does, and the kernel returns.  The next swa_plan_check
 * reports SWA_ERR_TIMEOUT (and clears the word); the context stays usable. */
swa_status swa_selftest_wait_timeout(swa_plan_t plan, uint64_t limit_ns, void* stream);

/* Self-test of the exponential the band kernel evaluates on the FMA pipe (an
 * addition of this library: the pages describe nothing like it).  For part of
 * the softmax exponentials the tensor-core kernel computes 2^x with a degree-3
 * polynomial instead of the MUFU unit; this entry point runs exactly that
 * device function on y[i] = 2^x[i], i < n (device pointers, fp32, enqueued on
 * `stream`), so that tests can hold it to its stated bound: relative error at
 * most 1.02e-4 for x in [-125.5, 128], a value in [0, 2^-125] below -125.5, and
 * exactly +0 for x <= -127 (and -inf).  SWA_ERR_INVALID_ARG for n < 0 or null
 * pointers with n > 0. */
swa_status swa_selftest_exp2_poly(const float* x, float* y, int n, void* stream);

/* Static, human-readable name of a status. */
const char* swa_status_string(swa_status s);

/* Transient-Global side keys / values: out[b,h,s,:] = mean of x[b,h,j,:] over the
 * tokens j of block s = [s*k, s*k + k) that are below valid_len[b]; the S =
 * floor(n / k) blocks cover the sequence, a trailing partial block joining the
 * last one; a block with no valid token is zero ("LongT5 长序列模型完全指南",
 * Transient-Global: tokens of each k-block are summed and normalised into one
 * global token; padding tokens belong to no block).  Device pointers, x [B,H,n,D],
 * out [B,H,floor(n/k),D], dtype bf16 or fp32, accumulation in fp32. */
swa_status swa_side_aggregate(const void* x, void* out, int batch, int heads, int seq_len,
                              int head_dim, int block, const int32_t* valid_len, swa_dtype dtype,
                              void* stream);

/* Host helper: T5 bidirectional relative-position bucket (32 buckets, max
 * distance 128) of delta = memory block - query block ("LongT5 长序列模型完全指南",
 * 相对位置编码 section and the LongT5Config defaults). */
int swa_relative_bucket(int delta);

/* Host helper: expand a per-head 32-bucket table [Hq][32] into the side-bias
 * table [Hq][S + nblk - 1] that swa_forward reads, column c holding the bucket of
 * delta = c - (nblk - 1).  Host pointers. */
swa_status swa_expand_side_bias(int num_q_heads, int num_side, int nblk, const float* table,
                                float* out);

/* ---------------------------------------------------------------------------
 * Allocation-free forward pass.  (An addition of this library: the pages
 * describe nothing like it.)
 *
 * For callers that cannot allocate memory when they run the attention: code
 * under a fixed memory budget or inside a host framework that owns all device
 * memory, real-time paths where allocating (and the synchronisation that a
 * device allocation can imply) is not allowed, and plug-ins that cannot keep a
 * plan object alive.  swa_forward_noalloc takes the plan descriptor directly and
 * runs the same kernels as swa_forward; it calls no cudaMalloc, cudaFree or any
 * other allocating routine, on the device or on the host.
 *
 * Its scratch memory (device error word, gathered global rows, split partials
 * of the global query rows) is one static device array of
 * SWA_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds until the
 * process exits.  The first call on a device looks up that array's device
 * address (cudaGetSymbolAddress, with the device current); make that first call
 * before any stream capture on the device.  Problems whose scratch would exceed
 * the limit -- only bf16 calls with global tokens need more than the error word
 * -- return SWA_ERR_UNSUPPORTED without launching anything.  All calls share the
 * array: each clears the error word and rewrites the rest before reading it, but
 * calls that overlap on the GPU (unordered streams or threads) race on it.
 * Arguments, layouts and the other statuses are those of swa_plan_create plus
 * swa_forward (desc: the plan descriptor; stream: a cudaStream_t); validation
 * and launches are shared with swa_forward.  With no plan there is no
 * swa_plan_check: outside SWA_DEBUG_CHECKS mode this entry point never
 * synchronises and cannot report an expired bounded wait (the next call clears
 * the error word); set SWA_DEBUG_CHECKS in desc->flags to have each call
 * synchronise and return SWA_ERR_TIMEOUT or SWA_ERR_DEVICE_CHECK.
 * ------------------------------------------------------------------------- */
#define SWA_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

swa_status swa_forward_noalloc(const swa_plan_desc* desc, const void* q, const void* k,
                               const void* v, const int32_t* global_idx, int num_global,
                               const void* side_k, const void* side_v, const float* bias,
                               const int32_t* window, const int32_t* dilation, int causal,
                               const int32_t* valid_len, void* out, float* lse, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SWA_H_ */
