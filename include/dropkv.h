/*
 * dropkv.h -- C ABI of libdropkv.so: DropKV prefill-time KV-cache eviction
 * scoring on NVIDIA B200 (sm_100a).
 *
 * What is computed (write-up "DropKV：精确单项输出扰动评分组件", section
 * 核心公式 "core formula", and the Algorithm 1 paragraph after it):
 *
 *   For each batch row b, KV head h and window query t (query head hq in the
 *   GQA group of h): the last `window` prompt positions are the queries; query
 *   t sits at position P_t = L_b - window + t and attends causally over keys
 *   0..P_t:  p = softmax(K q / sqrt(d)),  a = sum_j p_j v_j.
 *   Exact single-removal perturbation: Delta_j = p_j / (1 - p_j) * (a - v_j);
 *   s_j = sum over the window of ||Delta_j||^2.
 *   Scores of the query heads sharing a KV head are averaged (GQA mean-merge),
 *   max-pooled along the tokens (MaxPool1D), and the final window is set to
 *   +inf.  The lowest-scoring tokens are evicted.  A p_j that rounds to 1
 *   makes the removal singular: the call fails with DROPKV_ERR_SINGULAR, no
 *   epsilon is added.
 *
 * Conventions shared by every entry point:
 *   - All tensors are dense, row-major ("C-contiguous"), with the last index
 *     fastest.  Device pointers must be 16-byte aligned.  The caller owns every
 *     buffer; the library never allocates or frees device or pinned memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All device work is enqueued on it; nothing else is touched.
 *   - Arguments are validated on the host before anything is enqueued; a bad
 *     argument returns DROPKV_ERR_ARG and launches nothing.
 *   - There is no CPU fallback.  Without an sm_100 device current, compute
 *     calls return DROPKV_ERR_UNSUPPORTED.
 *   - The library is thread-safe as long as concurrent calls use different
 *     workspaces.
 */
#ifndef DROPKV_H_
#define DROPKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DROPKV_ABI_VERSION 2

#if defined(__GNUC__)
#define DROPKV_API __attribute__((visibility("default")))
#else
#define DROPKV_API
#endif

typedef enum dropkv_status {
  DROPKV_OK = 0,
  DROPKV_ERR_ARG = 1,          /* invalid shape, length, pointer, alignment or size     */
  DROPKV_ERR_SINGULAR = 2,     /* some p_j rounds to 1 in fp32 (1 - p_j is not > 0)      */
  DROPKV_ERR_CUDA = 3,         /* a CUDA runtime or driver call failed                   */
  DROPKV_ERR_UNSUPPORTED = 4,  /* no sm_100 device, or a path forced on a shape it lacks */
  DROPKV_ERR_WORKSPACE = 5,    /* workspace NULL or smaller than the query returned      */
  DROPKV_ERR_TIMEOUT = 6       /* a device-side wait gave up (bounded waits, no hang)    */
} dropkv_status;

typedef enum dropkv_dtype {
  DROPKV_BF16 = 0,  /* q, k, v stored as bfloat16; arithmetic in fp32 (tensor-core
                       operands bf16 with fp32 accumulation)                          */
  DROPKV_F32 = 1    /* q, k, v stored as float32; arithmetic in fp64 (CUDA cores)      */
} dropkv_dtype;

/* Which kernels compute the scores (dropkv_options.path). */
typedef enum dropkv_path {
  DROPKV_PATH_AUTO = 0,     /* tensor-core path when the shape allows it, else SIMT         */
  DROPKV_PATH_SIMT = 1,     /* fp32 CUDA-core kernels: any d <= 256, bf16 or f32            */
  DROPKV_PATH_TENSOR = 2    /* tcgen05 + TMA kernels: bf16, d == 128, G*window/chunks % 16 == 0 */
} dropkv_path;

/* Problem shape.  G = Hq / Hkv query heads share one KV head (query head hq
 * belongs to KV head hq / G).  window = number of observation queries w. */
typedef struct dropkv_shape {
  int32_t B;            /* batch rows, >= 1                                   */
  int32_t Hq;           /* query heads, a multiple of Hkv                     */
  int32_t Hkv;          /* KV heads, >= 1                                     */
  int32_t n_max;        /* padded cache length (row stride of k, v, scores)   */
  int32_t d;            /* head dimension, 1..256                             */
  int32_t window;       /* w >= 1; every length must satisfy w < L_b <= n_max */
  int32_t pool_kernel;  /* MaxPool1D kernel size: odd, 1..1023 (1 = no pooling) */
  int32_t dtype;        /* dropkv_dtype of q, k and v                         */
} dropkv_shape;

/* What is scored (dropkv_options.score). */
typedef enum dropkv_score {
  /* the exact single-removal output perturbation, sum over the window of
     ||p_j/(1-p_j) (a - v_j)||^2 (write-up section 核心公式); the default      */
  DROPKV_SCORE_PERTURBATION = 0,
  /* the attention-only negative control the write-up reports beside it
     (section 结果与独立对照): the attention mass sum_t p_j^(t) each token
     receives from the window queries.  Same merge, pooling, window protection
     and scores layout; never singular.  Only the first pass reads v (it
     still produces the window outputs); the second pass reads only k.       */
  DROPKV_SCORE_ATTENTION = 1
} dropkv_score;

/* Optional extras for dropkv_scores_ex.  Zero-initialise for defaults. */
typedef struct dropkv_options {
  int32_t path;        /* dropkv_path                                                  */
  int32_t score;       /* dropkv_score; other values are DROPKV_ERR_ARG                */
  float* attn_out;     /* device fp32 [B, Hq, w, d] or NULL: each window query's
                          attention output a (the write-up's result also returns the
                          window attention/output, section 代码映射与边界)              */
  float* stats_out;    /* device fp32 [B, Hq, w, 2] or NULL: (max logit, softmax
                          normaliser) per window query, logits scaled by 1/sqrt(d)   */
  void* const* events; /* NULL, or cudaEvent_t[n_events] owned by the caller: events
                          2i and 2i+1 are recorded on `stream` right before and after
                          the i-th kernel this call launches (for live timing)        */
  int32_t n_events;
  int32_t tc_ctas;     /* tensor path only: the most CTAs one scoring pass launches
                          per batch slice (0 = one per SM, at most 160).  Each CTA
                          walks a contiguous run of 128-token tiles of one (b, h,
                          query chunk), so fewer CTAs mean longer runs.  Values
                          below the slice's (b, h, chunk) unit count act as that
                          count, values above 160 as 160; < 0 is DROPKV_ERR_ARG.
                          Any value gives the same scores up to fp32 rounding.      */
} dropkv_options;

/* Bytes of device workspace dropkv_scores* needs for this shape (any lengths).
 * Returns 0 for an invalid shape. */
DROPKV_API size_t dropkv_scores_workspace_bytes(const dropkv_shape* shape);

/*
 * Score every cached token (write-up section 核心公式 and Algorithm 1 up to,
 * not including, the eviction itself).
 *   q        device [B, Hq, w, d]: the last w query rows of each sequence, in
 *            position order (row t belongs to position L_b - w + t).
 *   k, v     device [B, Hkv, n_max, d]: rows >= L_b are never read as data
 *            (they may hold anything, NaN included).
 *   lengths  HOST int32 [B] (L_b), or NULL for all n_max.
 *   scores   device fp32 [B, Hkv, n_max], written in full: merged+pooled scores
 *            for j < L_b - w, +inf for the window L_b - w <= j < L_b, NaN for
 *            j >= L_b.
 *   workspace / workspace_bytes: device scratch of at least
 *            dropkv_scores_workspace_bytes(shape) bytes, contents irrelevant.
 * Synchronises `stream` before returning so that it can report
 * DROPKV_ERR_SINGULAR; on that error the scores are unspecified.
 */
DROPKV_API dropkv_status dropkv_scores(const dropkv_shape* shape, const void* q, const void* k,
                            const void* v, const int32_t* lengths, float* scores,
                            void* workspace, size_t workspace_bytes, void* stream);

/* As dropkv_scores, without the synchronisation: returns once the work is
 * enqueued.  status_dev (device int32, caller-owned) receives DROPKV_OK, or
 * the largest error code the kernels raised (DROPKV_ERR_SINGULAR, or
 * DROPKV_ERR_TIMEOUT if a bounded device-side wait gave up), when the work
 * completes.  Host-side errors are returned directly and nothing is enqueued. */
DROPKV_API dropkv_status dropkv_scores_async(const dropkv_shape* shape, const void* q, const void* k,
                                  const void* v, const int32_t* lengths, float* scores,
                                  void* workspace, size_t workspace_bytes, void* stream,
                                  int32_t* status_dev);

/* dropkv_scores with options (kernel path choice, optional window outputs).
 * status_dev NULL => synchronous like dropkv_scores, else asynchronous. */
DROPKV_API dropkv_status dropkv_scores_ex(const dropkv_shape* shape, const void* q, const void* k,
                               const void* v, const int32_t* lengths, float* scores,
                               void* workspace, size_t workspace_bytes, void* stream,
                               int32_t* status_dev, const dropkv_options* options);

/* Bytes of device workspace dropkv_select needs.  0 for invalid sizes. */
DROPKV_API size_t dropkv_select_workspace_bytes(int32_t B, int32_t Hkv, int32_t n_max);

/*
 * Eviction (Algorithm 1's last step): for each (b, h) evict the
 * lengths[b] - keep_counts[b] tokens that come first in the order
 * (score ascending, position ascending); NaN orders above +inf.
 *   scores       device fp32 [B, Hkv, n_max] (only j < L_b is read).
 *   lengths      HOST int32 [B] or NULL (all n_max); keep_counts HOST int32 [B],
 *                0 <= keep_counts[b] <= lengths[b].
 *   keep_idx     device int32 [B, Hkv, max_keep]: kept positions ascending,
 *                then -1;  max_keep >= every keep_counts[b].
 *   evict_idx    device int32 [B, Hkv, max_evict]: evicted positions ascending,
 *                then -1;  max_evict >= every lengths[b] - keep_counts[b].
 *                (keep_idx / evict_idx may be NULL when max_keep / max_evict is 0.)
 * Asynchronous on `stream`; integer results are exact.  The CTAs of a
 * (b, h)'s cluster meet at hardware cluster barriers that every thread
 * reaches unconditionally, so the kernel has no wait that can give up; the
 * failure path (a wait that gives up, its (b, h)'s keep and evict slots all
 * -1, DROPKV_ERR_TIMEOUT) belongs to the bounded build that
 * dropkv_selftest_select_timeout runs.  Only dropkv_select_ex reports the
 * device status itself; this entry point enqueues nothing but the selection
 * kernel and leaves the workspace untouched.
 */
DROPKV_API dropkv_status dropkv_select(int32_t B, int32_t Hkv, int32_t n_max, const float* scores,
                            const int32_t* lengths, const int32_t* keep_counts,
                            int32_t* keep_idx, int32_t max_keep, int32_t* evict_idx,
                            int32_t max_evict, void* workspace, size_t workspace_bytes,
                            void* stream);

/* dropkv_select that reports the device-side status.  status_dev NULL: the
 * call synchronises `stream` and returns the kernels' status (DROPKV_OK, or
 * DROPKV_ERR_TIMEOUT from a build with bounded waits).  status_dev non-NULL
 * (device int32, 4-byte aligned, caller-owned): asynchronous; the call zeroes
 * *status_dev on the stream and the kernels raise it on an error.  Host-side
 * errors are returned directly and nothing is enqueued. */
DROPKV_API dropkv_status dropkv_select_ex(int32_t B, int32_t Hkv, int32_t n_max,
                                          const float* scores, const int32_t* lengths,
                                          const int32_t* keep_counts, int32_t* keep_idx,
                                          int32_t max_keep, int32_t* evict_idx, int32_t max_evict,
                                          void* workspace, size_t workspace_bytes, void* stream,
                                          int32_t* status_dev);

/*
 * dropkv_select without a workspace, for callers that cannot allocate device
 * memory (for example code inside a serving engine that owns all device memory
 * through its own pool, or a path that cannot afford cudaMalloc's implicit
 * device synchronisation).  The paper has no counterpart: this is an interface
 * variant of the eviction step above, with the same arguments minus the
 * workspace and the same results.
 *   Scratch: a 4 KiB array of static device memory inside the library, held by
 *   every GPU that loads the library until the process exits.  Sizes whose
 *   dropkv_select_workspace_bytes(min(B, 64), Hkv, n_max) exceeds 4 KiB would be
 *   rejected with DROPKV_ERR_WORKSPACE before anything is enqueued (the select
 *   path needs 256 bytes for any size, so none is).
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture.  No call allocates or frees memory.
 *   All calls share the array and it keeps the last call's contents: each
 *   call enqueues one memset of the array's 4-byte status word on `stream`
 *   before its kernels.  Calls whose work overlaps on the GPU, e.g. on
 *   two streams at once, race and must be serialised by the caller.
 *   The kernel's device status is not reported by this entry point (its
 *   status word sits in the shared array); use dropkv_select_ex where it
 *   must be read.
 */
DROPKV_API dropkv_status dropkv_select_noalloc(int32_t B, int32_t Hkv, int32_t n_max,
                                               const float* scores, const int32_t* lengths,
                                               const int32_t* keep_counts, int32_t* keep_idx,
                                               int32_t max_keep, int32_t* evict_idx,
                                               int32_t max_evict, void* stream);

/*
 * Scoring and eviction in one call (write-up section 核心公式 and the whole of
 * Algorithm 1): the work of dropkv_scores_ex followed by dropkv_select_ex on
 * its scores, with the same results -- `scores` written exactly as
 * dropkv_scores writes them, and the same keep / evict lists -- enqueued by
 * one call (each batch slice of up to 64 rows is scored and then selected).
 *   Arguments as dropkv_scores_ex (shape, q, k, v, lengths, scores,
 *   workspace of dropkv_scores_workspace_bytes(shape) bytes, stream, options)
 *   and dropkv_select (keep_counts, keep_idx, max_keep, evict_idx, max_evict).
 *   status_dev NULL: synchronous; returns DROPKV_ERR_SINGULAR or
 *   DROPKV_ERR_TIMEOUT when the kernels raised one.  status_dev non-NULL
 *   (device int32, caller-owned): asynchronous; *status_dev receives the
 *   largest code the kernels raised.  Host-side errors are returned directly
 *   and nothing is enqueued.  On DROPKV_ERR_SINGULAR the scores and lists are
 *   unspecified.
 */
DROPKV_API dropkv_status dropkv_scores_select(const dropkv_shape* shape, const void* q,
                                              const void* k, const void* v,
                                              const int32_t* lengths, const int32_t* keep_counts,
                                              float* scores, int32_t* keep_idx, int32_t max_keep,
                                              int32_t* evict_idx, int32_t max_evict,
                                              void* workspace, size_t workspace_bytes,
                                              void* stream, int32_t* status_dev,
                                              const dropkv_options* options);

/* Which path DROPKV_PATH_AUTO picks for this shape (DROPKV_PATH_SIMT or
 * DROPKV_PATH_TENSOR); no device needed.  Returns -1 for an invalid shape. */
DROPKV_API int32_t dropkv_auto_path(const dropkv_shape* shape);

/* Number of kernels one dropkv_scores / dropkv_select call launches for this
 * shape and lengths (host-only planning, no device needed); -1 if invalid. */
DROPKV_API int32_t dropkv_scores_launches(const dropkv_shape* shape, const int32_t* lengths,
                               int32_t path);
DROPKV_API int32_t dropkv_select_launches(int32_t B, int32_t Hkv, int32_t n_max, const int32_t* lengths);
/* Kernel launches of one dropkv_scores_select call (-1 for an invalid shape). */
DROPKV_API int32_t dropkv_scores_select_launches(const dropkv_shape* shape, const int32_t* lengths,
                                                 int32_t path);

/* Static description of a status code. */
DROPKV_API const char* dropkv_status_string(dropkv_status status);

/* The cudaError_t code (as an int) behind the last DROPKV_ERR_CUDA that a call
 * made on this host thread returned, and its name; 0 / "cudaSuccess" before
 * any.  Host-only, never fails. */
DROPKV_API int32_t dropkv_last_cuda_error(void);
DROPKV_API const char* dropkv_last_cuda_error_string(void);

/* Self-test of the bounded device waits that the kernels use: enqueues one
 * CTA on `stream` that waits on an mbarrier nothing ever arrives on, gives up
 * after limit_ns nanoseconds of %globaltimer and then writes
 * DROPKV_ERR_TIMEOUT into *status_dev (device int32, 4-byte aligned, not
 * cleared by the call).  The kernel returns normally: no fault or trap, the
 * context stays usable.  0 < limit_ns <= 1e9, else DROPKV_ERR_ARG; no
 * sm_100 device gives DROPKV_ERR_UNSUPPORTED. */
DROPKV_API dropkv_status dropkv_selftest_wait_timeout(int32_t* status_dev, uint64_t limit_ns,
                                                      void* stream);

/* Self-test of the select kernel's failure path: runs the select of
 * dropkv_select on the given arguments (B <= 64) in its bounded build (the
 * radix rounds separated by mbarrier phases with bounded waits instead of
 * hardware cluster barriers) with one CTA of every segment's cluster
 * withholding its arrivals of the first radix round (so the other CTAs'
 * waits for them run out) and every bounded wait limited to limit_ns
 * nanoseconds (0 < limit_ns <= 1e9).  Every segment with
 * at least one eviction then ends with DROPKV_ERR_TIMEOUT in *status_dev
 * (device int32, zeroed by the call) and all its keep and evict slots set to
 * -1.  Asynchronous on `stream`; no fault or trap is involved and the context
 * stays usable.  Errors as for dropkv_select, plus DROPKV_ERR_ARG for B > 64
 * or a bad status_dev / limit. */
DROPKV_API dropkv_status dropkv_selftest_select_timeout(int32_t B, int32_t Hkv, int32_t n_max,
                                                        const float* scores,
                                                        const int32_t* lengths,
                                                        const int32_t* keep_counts,
                                                        int32_t* keep_idx, int32_t max_keep,
                                                        int32_t* evict_idx, int32_t max_evict,
                                                        int32_t* status_dev, uint64_t limit_ns,
                                                        void* stream);

/* DROPKV_ABI_VERSION of the loaded library. */
DROPKV_API int32_t dropkv_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DROPKV_H_ */
