// api.cu -- the extern "C" entry points of libdropkv.so: argument checks,
// workspace carve-up, batch slicing and the launch sequence.  No device memory
// is ever allocated here; every launch goes to the caller's stream.
#include <math.h>
#include <string.h>

#include "internal.h"

namespace dropkv {

namespace {

constexpr size_t kAlign = 256;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int32_t length_of(const dropkv_shape& s, const int32_t* lengths, int b) {
  return lengths ? lengths[b] : s.n_max;
}

dropkv_status validate_shape(const dropkv_shape* sp, const int32_t* lengths) {
  if (!sp) return DROPKV_ERR_ARG;
  const dropkv_shape& s = *sp;
  if (s.B < 1 || s.Hq < 1 || s.Hkv < 1 || s.Hq % s.Hkv != 0) return DROPKV_ERR_ARG;
  if (s.d < 1 || s.d > 256) return DROPKV_ERR_ARG;
  if (s.window < 1 || s.n_max <= s.window) return DROPKV_ERR_ARG;
  if (s.pool_kernel < 1 || s.pool_kernel % 2 == 0 || s.pool_kernel > 1023) return DROPKV_ERR_ARG;
  if (s.dtype != DROPKV_BF16 && s.dtype != DROPKV_F32) return DROPKV_ERR_ARG;
  // every buffer index must fit comfortably in 63 bits
  const double elems = (double)s.B * s.Hkv * (double)s.n_max * s.d;
  if (elems > 4.0e18) return DROPKV_ERR_ARG;
  if ((double)s.Hq * s.window > 1.0e9) return DROPKV_ERR_ARG;
  if (lengths)
    for (int b = 0; b < s.B; ++b)
      if (lengths[b] <= s.window || lengths[b] > s.n_max) return DROPKV_ERR_ARG;
  return DROPKV_OK;
}

dropkv_status check_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return DROPKV_ERR_UNSUPPORTED;
  }
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return DROPKV_ERR_UNSUPPORTED;
  }
  if (major != 10 || minor != 0) return DROPKV_ERR_UNSUPPORTED;  // built for sm_100a only
  return DROPKV_OK;
}

int resolve_path(const dropkv_shape& s, int requested) {
  if (requested == DROPKV_PATH_SIMT) return DROPKV_PATH_SIMT;
  if (requested == DROPKV_PATH_TENSOR) return tc_shape_ok(s) ? DROPKV_PATH_TENSOR : -1;
  if (requested == DROPKV_PATH_AUTO) return tc_shape_ok(s) ? DROPKV_PATH_TENSOR : DROPKV_PATH_SIMT;
  return -2;
}

}  // namespace

dropkv_status device_ok() { return check_device(); }

// Tensor path: bf16, d = 128, and the G*w query rows of a KV head split into
// equal chunks whose widths suit the token-major second passes' MMAs.
bool tc_shape_ok(const dropkv_shape& s) {
  if (!tc_available()) return false;
  if (s.dtype != DROPKV_BF16 || s.d != 128 || s.n_max < 128) return false;
  const int nq = (s.Hq / s.Hkv) * s.window;
  // the single-CTA second pass: chunks of <= 128 rows, multiples of 16; the
  // pair second pass: chunks of <= 256 rows taken as one or two halves whose
  // width (the MMA's N) is a multiple of 16
  const int chunks = (nq + 127) / 128, chunks2 = (nq + 255) / 256;
  if (nq % (16 * chunks) != 0 || nq % chunks2 != 0) return false;
  const int nqc2 = nq / chunks2;
  if (nqc2 % (nqc2 > 128 ? 32 : 16) != 0) return false;
  return true;
}

TcPlan tc_plan(const dropkv_shape& s) {
  TcPlan p;
  const int nq = (s.Hq / s.Hkv) * s.window;
  p.chunks = (nq + 127) / 128;
  p.nqc = nq / p.chunks;
  p.chunks1 = (nq + 255) / 256;
  p.rows1 = (nq + p.chunks1 - 1) / p.chunks1;
  p.chunks2 = (nq + 255) / 256;
  p.nqc2 = nq / p.chunks2;
  return p;
}

ScoresLayout scores_layout(const dropkv_shape& s, int Bs) {
  ScoresLayout l;
  const size_t rows = (size_t)Bs * s.Hq * s.window;
  const bool tc = tc_shape_ok(s);
  // tensor path: four column groups per query chunk of either second pass
  l.nparts = tc ? 4 * tc_plan(s).chunks : 1;
  size_t o = 0;
  l.status = o;
  o += kAlign;
  l.stats = o;
  o = align_up(o + rows * 2 * sizeof(double), kAlign);
  l.attn = o;
  o = align_up(o + rows * s.d * sizeof(double), kAlign);
  l.parts = o;
  o = align_up(o + (size_t)l.nparts * Bs * s.Hkv * (size_t)s.n_max * sizeof(float), kAlign);
  l.tc_partial = l.tc_ahi = l.tc_alo = l.tc_qstat = l.tc_nv = l.tc_tmin = o;
  if (tc) {
    const TcPlan p = tc_plan(s);
    // pass-1 partials: at most (split target + one per (b, h, chunk)) CTAs,
    // rows1 rows each of (a[128], max, normaliser, pad).
    const size_t ctas = (size_t)tc_split_target() + (size_t)Bs * s.Hkv * p.chunks1;
    l.tc_partial = o;
    o = align_up(o + ctas * p.rows1 * kTcPartStride * sizeof(float), kAlign);
    l.tc_ahi = o;
    o = align_up(o + rows * s.d * 2, kAlign);
    l.tc_alo = o;
    o = align_up(o + rows * s.d * 2, kAlign);
    l.tc_qstat = o;
    o = align_up(o + rows * 4 * sizeof(float), kAlign);
    l.tc_nv = o;  // per head padded to whole 128-token tiles (512-byte rows per tile)
    o = align_up(o + (size_t)Bs * s.Hkv * (size_t)((s.n_max + 127) / 128) * 128 * sizeof(float),
                 kAlign);
    l.tc_tmin = o;
    o = align_up(o + (size_t)Bs * s.Hkv * (size_t)((s.n_max + 127) / 128) * p.chunks1 * sizeof(float),
                 kAlign);
  }
  l.total = o;
  return l;
}

// The CUDA error behind the last DROPKV_ERR_CUDA returned to this thread.
static thread_local cudaError_t g_last_cuda = cudaSuccess;
dropkv_status cuda_fail(cudaError_t e) {
  g_last_cuda = e == cudaSuccess ? cudaErrorUnknown : e;
  return DROPKV_ERR_CUDA;
}

dropkv_status check_select_args(int32_t B, int32_t Hkv, int32_t n_max, const float* scores,
                                const int32_t* lengths, const int32_t* keep_counts,
                                const int32_t* keep_idx, int32_t max_keep,
                                const int32_t* evict_idx, int32_t max_evict) {
  if (B < 1 || Hkv < 1 || n_max < 1 || !scores || !keep_counts) return DROPKV_ERR_ARG;
  if ((!keep_idx && max_keep > 0) || (!evict_idx && max_evict > 0)) return DROPKV_ERR_ARG;
  if (max_keep < 0 || max_evict < 0) return DROPKV_ERR_ARG;
  if (!aligned16(scores) || ((uintptr_t)keep_idx & 3u) || ((uintptr_t)evict_idx & 3u))
    return DROPKV_ERR_ARG;
  if ((double)B * Hkv * (double)n_max > 4.0e18) return DROPKV_ERR_ARG;
  for (int b = 0; b < B; ++b) {
    const int L = lengths ? lengths[b] : n_max;
    if (L < 0 || L > n_max) return DROPKV_ERR_ARG;
    if (keep_counts[b] < 0 || keep_counts[b] > L) return DROPKV_ERR_ARG;
    if (keep_counts[b] > max_keep || L - keep_counts[b] > max_evict) return DROPKV_ERR_ARG;
  }
  return DROPKV_OK;
}

dropkv_status run_select(int32_t B, int32_t Hkv, int32_t n_max, const float* scores,
                         const int32_t* lengths, const int32_t* keep_counts, int32_t* keep_idx,
                         int32_t max_keep, int32_t* evict_idx, int32_t max_evict,
                         int32_t* status_word, cudaStream_t st) {
  // one reset per call: a timeout in one launch slice stays visible after the
  // next (status_word NULL: the caller does not ask for the device status)
  if (status_word)
    if (cudaError_t e = cudaMemsetAsync(status_word, 0, sizeof(int32_t), st)) return cuda_fail(e);
  for (int b0 = 0; b0 < B; b0 += kMaxB) {
    const int Bs = (B - b0) < kMaxB ? (B - b0) : kMaxB;
    int32_t L[kMaxB], K[kMaxB];
    for (int i = 0; i < Bs; ++i) {
      L[i] = lengths ? lengths[b0 + i] : n_max;
      K[i] = keep_counts[b0 + i];
    }
    const size_t seg0 = (size_t)b0 * Hkv;
    cudaError_t e = launch_select(Bs, Hkv, n_max, scores + seg0 * n_max, L, K,
                                  keep_idx + seg0 * max_keep, max_keep,
                                  evict_idx + seg0 * max_evict, max_evict, status_word, st);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return DROPKV_OK;
}

// The selection dropkv_scores_select adds to the scoring call.
struct SelectSpec {
  const int32_t* keep_counts;
  int32_t* keep_idx;
  int32_t max_keep;
  int32_t* evict_idx;
  int32_t max_evict;
};

// Runs the scoring pipeline, and after each batch slice's scores its
// selection when `sel` is given; `sync` selects the synchronous contract.
static dropkv_status run_scores(const dropkv_shape* sp, const void* q, const void* k,
                                const void* v, const int32_t* lengths, float* scores,
                                void* workspace, size_t ws_bytes, void* stream,
                                int32_t* status_dev, const dropkv_options* opt, bool sync,
                                const SelectSpec* sel = nullptr) {
  dropkv_status r = validate_shape(sp, lengths);
  if (r != DROPKV_OK) return r;
  const dropkv_shape& s = *sp;
  if (!q || !k || !v || !scores) return DROPKV_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(scores)) return DROPKV_ERR_ARG;
  if (status_dev && ((uintptr_t)status_dev & 3u)) return DROPKV_ERR_ARG;
  if (opt && opt->attn_out && !aligned16(opt->attn_out)) return DROPKV_ERR_ARG;
  if (opt && opt->stats_out && !aligned16(opt->stats_out)) return DROPKV_ERR_ARG;
  const int score = opt ? opt->score : DROPKV_SCORE_PERTURBATION;
  if (score != DROPKV_SCORE_PERTURBATION && score != DROPKV_SCORE_ATTENTION) return DROPKV_ERR_ARG;
  const int tc_ctas = opt ? opt->tc_ctas : 0;
  if (tc_ctas < 0) return DROPKV_ERR_ARG;
  const int path = resolve_path(s, opt ? opt->path : DROPKV_PATH_AUTO);
  if (path == -2) return DROPKV_ERR_ARG;
  if (path == -1) return DROPKV_ERR_UNSUPPORTED;
  if (sel) {
    r = check_select_args(s.B, s.Hkv, s.n_max, scores, lengths, sel->keep_counts, sel->keep_idx,
                          sel->max_keep, sel->evict_idx, sel->max_evict);
    if (r != DROPKV_OK) return r;
  }
  const size_t need = dropkv_scores_workspace_bytes(sp);
  if (!workspace || ws_bytes < need || !aligned16(workspace)) return DROPKV_ERR_WORKSPACE;
  r = check_device();
  if (r != DROPKV_OK) return r;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* ws = reinterpret_cast<char*>(workspace);
  const int Bs_max = s.B < kMaxB ? s.B : kMaxB;
  const ScoresLayout lay = scores_layout(s, Bs_max);
  int32_t* status_word = status_dev ? status_dev : reinterpret_cast<int32_t*>(ws + lay.status);
  if (cudaError_t e0 = cudaMemsetAsync(status_word, 0, sizeof(int32_t), st)) return cuda_fail(e0);

  KernelEvents kev;
  if (opt && opt->events && opt->n_events > 0) {
    kev.ev = opt->events;
    kev.n = opt->n_events;
  }
  const size_t esz = s.dtype == DROPKV_BF16 ? 2 : 4;
  for (int b0 = 0; b0 < s.B; b0 += kMaxB) {
    const int Bs = (s.B - b0) < kMaxB ? (s.B - b0) : kMaxB;
    Lens lens;
    lens.B = Bs;
    for (int i = 0; i < Bs; ++i) lens.L[i] = length_of(s, lengths, b0 + i);
    const size_t qoff = (size_t)b0 * s.Hq * s.window * s.d;
    const size_t kvoff = (size_t)b0 * s.Hkv * (size_t)s.n_max * s.d;
    const char* qs = reinterpret_cast<const char*>(q) + qoff * esz;
    const char* ks = reinterpret_cast<const char*>(k) + kvoff * esz;
    const char* vs = reinterpret_cast<const char*>(v) + kvoff * esz;
    float* sc = scores + (size_t)b0 * s.Hkv * s.n_max;
    float* attn_user = (opt && opt->attn_out) ? opt->attn_out + qoff : nullptr;
    float* stats_user =
        (opt && opt->stats_out) ? opt->stats_out + (size_t)b0 * s.Hq * s.window * 2 : nullptr;
    double* stats_ws = reinterpret_cast<double*>(ws + lay.stats);
    void* attn_ws = ws + lay.attn;
    float* parts = reinterpret_cast<float*>(ws + lay.parts);
    const size_t part_stride = (size_t)Bs * s.Hkv * s.n_max;
    int nparts = path == DROPKV_PATH_SIMT ? 1 : lay.nparts;
    cudaError_t e;
    if (path == DROPKV_PATH_SIMT) {
      kev.begin(st);
      e = launch_simt_pass1(s, qs, ks, vs, lens, stats_ws, attn_ws, stats_user, attn_user, st);
      kev.end(st);
      if (e == cudaSuccess) {
        kev.begin(st);
        e = launch_simt_pass2(s, qs, ks, vs, lens, stats_ws, attn_ws, parts, status_word, score,
                              st);
        kev.end(st);
      }
    } else {
      e = launch_tc_scores(s, qs, ks, vs, lens, lay, ws, attn_user, stats_user, status_word, score,
                           tc_ctas, st, kev, &nparts);
    }
    if (e == cudaSuccess) {
      kev.begin(st);
      e = launch_epilogue(s, lens, parts, nparts, part_stride, sc, st);
      kev.end(st);
    }
    if (e == cudaSuccess && sel) {  // the selection of this slice's rows
      const size_t seg0 = (size_t)b0 * s.Hkv;
      kev.begin(st);
      e = launch_select(Bs, s.Hkv, s.n_max, sc, lens.L, sel->keep_counts + b0,
                        sel->keep_idx + seg0 * sel->max_keep, sel->max_keep,
                        sel->evict_idx + seg0 * sel->max_evict, sel->max_evict, status_word, st);
      kev.end(st);
    }
    if (e != cudaSuccess) return e == cudaErrorNotSupported ? DROPKV_ERR_UNSUPPORTED : cuda_fail(e);
  }
  if (!sync) return DROPKV_OK;
  int32_t host_status = 0;
  if (cudaError_t e1 =
          cudaMemcpyAsync(&host_status, status_word, sizeof(int32_t), cudaMemcpyDeviceToHost, st))
    return cuda_fail(e1);
  if (cudaError_t e2 = cudaStreamSynchronize(st)) return cuda_fail(e2);
  if (host_status != 0) return static_cast<dropkv_status>(host_status);
  return DROPKV_OK;
}

}  // namespace dropkv

using namespace dropkv;

extern "C" {

size_t dropkv_scores_workspace_bytes(const dropkv_shape* shape) {
  if (validate_shape(shape, nullptr) != DROPKV_OK) return 0;
  const int Bs = shape->B < kMaxB ? shape->B : kMaxB;
  return scores_layout(*shape, Bs).total;
}

dropkv_status dropkv_scores(const dropkv_shape* shape, const void* q, const void* k,
                            const void* v, const int32_t* lengths, float* scores,
                            void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange range("dropkv_scores");
  return run_scores(shape, q, k, v, lengths, scores, workspace, workspace_bytes, stream, nullptr,
                    nullptr, true);
}

dropkv_status dropkv_scores_async(const dropkv_shape* shape, const void* q, const void* k,
                                  const void* v, const int32_t* lengths, float* scores,
                                  void* workspace, size_t workspace_bytes, void* stream,
                                  int32_t* status_dev) {
  NvtxRange range("dropkv_scores_async");
  if (!status_dev) return DROPKV_ERR_ARG;
  return run_scores(shape, q, k, v, lengths, scores, workspace, workspace_bytes, stream,
                    status_dev, nullptr, false);
}

dropkv_status dropkv_scores_ex(const dropkv_shape* shape, const void* q, const void* k,
                               const void* v, const int32_t* lengths, float* scores,
                               void* workspace, size_t workspace_bytes, void* stream,
                               int32_t* status_dev, const dropkv_options* options) {
  NvtxRange range("dropkv_scores_ex");
  return run_scores(shape, q, k, v, lengths, scores, workspace, workspace_bytes, stream,
                    status_dev, options, status_dev == nullptr);
}

dropkv_status dropkv_scores_select(const dropkv_shape* shape, const void* q, const void* k,
                                   const void* v, const int32_t* lengths,
                                   const int32_t* keep_counts, float* scores, int32_t* keep_idx,
                                   int32_t max_keep, int32_t* evict_idx, int32_t max_evict,
                                   void* workspace, size_t workspace_bytes, void* stream,
                                   int32_t* status_dev, const dropkv_options* options) {
  NvtxRange range("dropkv_scores_select");
  if (!shape) return DROPKV_ERR_ARG;
  const SelectSpec sel = {keep_counts, keep_idx, max_keep, evict_idx, max_evict};
  return run_scores(shape, q, k, v, lengths, scores, workspace, workspace_bytes, stream,
                    status_dev, options, status_dev == nullptr, &sel);
}

size_t dropkv_select_workspace_bytes(int32_t B, int32_t Hkv, int32_t n_max) {
  if (B < 1 || Hkv < 1 || n_max < 1) return 0;
  const int Bs = B < kMaxB ? B : kMaxB;
  return select_workspace_bytes(Bs, Hkv, n_max);
}

static dropkv_status select_entry(int32_t B, int32_t Hkv, int32_t n_max, const float* scores,
                                  const int32_t* lengths, const int32_t* keep_counts,
                                  int32_t* keep_idx, int32_t max_keep, int32_t* evict_idx,
                                  int32_t max_evict, void* workspace, size_t workspace_bytes,
                                  void* stream, int32_t* status_dev, bool sync) {
  dropkv_status r = check_select_args(B, Hkv, n_max, scores, lengths, keep_counts, keep_idx,
                                      max_keep, evict_idx, max_evict);
  if (r != DROPKV_OK) return r;
  if (status_dev && ((uintptr_t)status_dev & 3u)) return DROPKV_ERR_ARG;
  const size_t need = dropkv_select_workspace_bytes(B, Hkv, n_max);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return DROPKV_ERR_WORKSPACE;
  r = check_device();
  if (r != DROPKV_OK) return r;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the plain entry point reports no device status: nothing to reset or record
  int32_t* status_word =
      status_dev ? status_dev : (sync ? reinterpret_cast<int32_t*>(workspace) : nullptr);
  r = run_select(B, Hkv, n_max, scores, lengths, keep_counts, keep_idx, max_keep, evict_idx,
                 max_evict, status_word, st);
  if (r != DROPKV_OK || !sync) return r;
  int32_t host_status = 0;
  if (cudaError_t e1 =
          cudaMemcpyAsync(&host_status, status_word, sizeof(int32_t), cudaMemcpyDeviceToHost, st))
    return cuda_fail(e1);
  if (cudaError_t e2 = cudaStreamSynchronize(st)) return cuda_fail(e2);
  return host_status != 0 ? static_cast<dropkv_status>(host_status) : DROPKV_OK;
}

dropkv_status dropkv_select(int32_t B, int32_t Hkv, int32_t n_max, const float* scores,
                            const int32_t* lengths, const int32_t* keep_counts,
                            int32_t* keep_idx, int32_t max_keep, int32_t* evict_idx,
                            int32_t max_evict, void* workspace, size_t workspace_bytes,
                            void* stream) {
  NvtxRange range("dropkv_select");
  return select_entry(B, Hkv, n_max, scores, lengths, keep_counts, keep_idx, max_keep, evict_idx,
                      max_evict, workspace, workspace_bytes, stream, nullptr, false);
}

dropkv_status dropkv_select_ex(int32_t B, int32_t Hkv, int32_t n_max, const float* scores,
                               const int32_t* lengths, const int32_t* keep_counts,
                               int32_t* keep_idx, int32_t max_keep, int32_t* evict_idx,
                               int32_t max_evict, void* workspace, size_t workspace_bytes,
                               void* stream, int32_t* status_dev) {
  NvtxRange range("dropkv_select_ex");
  return select_entry(B, Hkv, n_max, scores, lengths, keep_counts, keep_idx, max_keep, evict_idx,
                      max_evict, workspace, workspace_bytes, stream, status_dev,
                      status_dev == nullptr);
}

int32_t dropkv_auto_path(const dropkv_shape* shape) {
  if (validate_shape(shape, nullptr) != DROPKV_OK) return -1;
  return tc_shape_ok(*shape) ? DROPKV_PATH_TENSOR : DROPKV_PATH_SIMT;
}

int32_t dropkv_scores_launches(const dropkv_shape* shape, const int32_t* lengths, int32_t path) {
  if (validate_shape(shape, lengths) != DROPKV_OK) return -1;
  const int p = resolve_path(*shape, path);
  if (p < 0) return -1;
  const int slices = (shape->B + kMaxB - 1) / kMaxB;
  const int per = (p == DROPKV_PATH_SIMT) ? 3 : tc_launch_count() + 1;
  return slices * per;
}

int32_t dropkv_scores_select_launches(const dropkv_shape* shape, const int32_t* lengths,
                                      int32_t path) {
  const int32_t n = dropkv_scores_launches(shape, lengths, path);
  if (n < 0) return -1;
  return n + ((shape->B + kMaxB - 1) / kMaxB) * select_launch_count();
}

int32_t dropkv_select_launches(int32_t B, int32_t Hkv, int32_t n_max, const int32_t* lengths) {
  (void)lengths;
  if (B < 1 || Hkv < 1 || n_max < 1) return -1;
  return ((B + kMaxB - 1) / kMaxB) * select_launch_count();
}

int32_t dropkv_last_cuda_error(void) { return (int32_t)g_last_cuda; }
const char* dropkv_last_cuda_error_string(void) { return cudaGetErrorName(g_last_cuda); }

const char* dropkv_status_string(dropkv_status status) {
  switch (status) {
    case DROPKV_OK: return "ok";
    case DROPKV_ERR_ARG: return "invalid argument";
    case DROPKV_ERR_SINGULAR: return "singular input: some p_j rounds to 1";
    case DROPKV_ERR_CUDA: return "CUDA error";
    case DROPKV_ERR_UNSUPPORTED: return "unsupported device or shape";
    case DROPKV_ERR_WORKSPACE: return "workspace missing or too small";
    case DROPKV_ERR_TIMEOUT: return "a device-side wait timed out";
  }
  return "unknown status";
}

int32_t dropkv_abi_version(void) { return DROPKV_ABI_VERSION; }

}  // extern "C"
