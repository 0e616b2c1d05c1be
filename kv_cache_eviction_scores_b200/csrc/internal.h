// internal.h -- host-side declarations shared by the libdropkv.so sources.
#pragma once

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stddef.h>
#include <stdint.h>

#include "dropkv.h"

namespace dropkv {

// An NVTX range named after a C entry point, held over its argument checks
// and launches, so that a timeline tool (or ncu's --nvtx-include filter) can
// attribute the kernels to the call.  NVTX is header-only: with no tool
// attached a push / pop pair is a call through a no-op function pointer.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Batch rows handled per launch; larger batches are processed in slices.
constexpr int kMaxB = 64;

// Bits of the device status word (the value equals DROPKV_ERR_SINGULAR).
constexpr int kStatusSingular = DROPKV_ERR_SINGULAR;

// Per-slice sequence lengths, passed by value as a kernel parameter.
struct Lens {
  int32_t B;
  int32_t L[kMaxB];
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Optional caller-owned CUDA events recorded around each kernel launch.
struct KernelEvents {
  void* const* ev = nullptr;
  int n = 0;
  int i = 0;
  void begin(cudaStream_t st) {
    if (ev && 2 * i + 1 < n) cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev[2 * i]), st);
  }
  void end(cudaStream_t st) {
    if (ev && 2 * i + 1 < n) cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev[2 * i + 1]), st);
    ++i;
  }
};

// Launches `kern` on `st`; with pdl = true the launch carries the programmatic
// stream-serialization attribute, so that it may overlap the tail of the
// previous kernel in the stream (the kernel must call pdl_wait() before it
// reads that kernel's results).  cluster_x > 1 launches clusters of that size.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t st, bool pdl, int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = (unsigned)cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = n ? attr : nullptr;
  cfg.numAttrs = (unsigned)n;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// ---- scoring: workspace carve-up ------------------------------------------
struct ScoresLayout {
  size_t status;     // int32 status word (sync variant)
  size_t stats;      // fp64 [B, Hq, w, 2]  (max logit, normaliser), SIMT path
  size_t attn;       // [B, Hq, w, d] window attention output a (8 bytes per element)
  size_t parts;      // fp32 [nparts][B, Hkv, n_max] partial merged scores
  size_t tc_partial; // fp32 pass-1 split partials (tensor path)
  size_t tc_ahi;     // bf16 [B, Hq, w, d] high part of a (tensor path)
  size_t tc_alo;     // bf16 [B, Hq, w, d] low part of a (tensor path)
  size_t tc_qstat;   // fp32 [B, Hq, w, 4] per-query pass-2 constants (tensor path)
  size_t tc_nv;      // fp32 [B, Hkv, ceil(n_max/128)*128] ||v_j||^2 (tensor path, pass 1 -> pass 2)
  size_t tc_tmin;    // fp32 [B, Hkv, ceil(n_max/128), chunks1] min ||v_j||^2 per tile share
  size_t total;
  int nparts;
};

// Tensor-path plan for one batch slice.
struct TcPlan {
  int chunks;        // pass-2 query chunks per KV head (G*w split into chunks of nqc rows)
  int nqc;           // rows per pass-2 chunk (multiple of 16, <= 128)
  int chunks1;       // pass-1 query chunks per KV head (two 128-row query tiles each)
  int rows1;         // rows per pass-1 chunk (<= 256; the last chunk may be shorter)
  int chunks2;       // CTA-pair pass-2 query chunks per KV head
  int nqc2;          // rows per pair chunk (multiple of 16, <= 256)
};
// floats per pass-1 partial row: O[128], max, normaliser, padding
constexpr int kTcPartStride = 132;

bool tc_shape_ok(const dropkv_shape& s);
// DROPKV_OK when the current device is an sm_100 part the kernels run on.
dropkv_status device_ok();
TcPlan tc_plan(const dropkv_shape& s);
ScoresLayout scores_layout(const dropkv_shape& s, int B_slice);

// ---- launchers (each returns the CUDA error of its launch) ----------------
// SIMT path.  stats_ws: fp64 [rows][2]; attn_ws: [rows][d] in the path's
// arithmetic type (fp32 for bf16 inputs, fp64 for fp32 inputs); the *_user
// pointers (optional) receive fp32 copies.
cudaError_t launch_simt_pass1(const dropkv_shape& s, const void* q, const void* k,
                              const void* v, const Lens& lens, double* stats_ws, void* attn_ws,
                              float* stats_user, float* attn_user, cudaStream_t st);
cudaError_t launch_simt_pass2(const dropkv_shape& s, const void* q, const void* k,
                              const void* v, const Lens& lens, const double* stats_ws,
                              const void* attn_ws, float* part, int32_t* status, int score,
                              cudaStream_t st);
cudaError_t launch_epilogue(const dropkv_shape& s, const Lens& lens, const float* parts,
                            int nparts, size_t part_stride, float* scores, cudaStream_t st);

// Tensor-core path (tcgen05 + TMA); returns cudaErrorNotSupported when the
// tensor maps cannot be encoded.  *nparts_used receives how many partial-score
// planes per (b, h) the second pass wrote (the epilogue sums them).
// cta_budget: most CTAs per pass (0 = one per SM).
cudaError_t launch_tc_scores(const dropkv_shape& s, const void* q, const void* k,
                             const void* v, const Lens& lens, const ScoresLayout& lay,
                             char* ws, float* attn_out, float* stats_out, int32_t* status,
                             int score, int cta_budget, cudaStream_t st, KernelEvents& kev,
                             int* nparts_used);
int tc_launch_count();
int tc_split_target();
bool tc_available();

// ---- selection --------------------------------------------------------------
size_t select_workspace_bytes(int B, int Hkv, int n_max);
int select_launch_count();
// One launch slice (B <= kMaxB rows).  `status` (device int32) receives
// DROPKV_ERR_TIMEOUT by atomicMax if a bounded wait gives up; the caller
// zeroes it once per call.
cudaError_t launch_select(int B, int Hkv, int n_max, const float* scores, const int32_t* L,
                          const int32_t* keep, int32_t* keep_idx, int32_t max_keep,
                          int32_t* evict_idx, int32_t max_evict, int32_t* status,
                          cudaStream_t st);

// The same launch for the select self-test: CTA rank 1 of every segment's
// cluster withholds its arrivals of the first round and every bounded wait
// gives up after wait_ns, so the segments with evictions end in
// DROPKV_ERR_TIMEOUT.
cudaError_t launch_select_stalled(int B, int Hkv, int n_max, const float* scores,
                                  const int32_t* L, const int32_t* keep, int32_t* keep_idx,
                                  int32_t max_keep, int32_t* evict_idx, int32_t max_evict,
                                  int32_t* status, uint64_t wait_ns, cudaStream_t st);

// Shared by the select entry points: host-side argument checks, and the
// slice loop with one status reset per call (returns DROPKV_ERR_CUDA through
// cuda_fail, which records the CUDA error for dropkv_last_cuda_error).
dropkv_status check_select_args(int32_t B, int32_t Hkv, int32_t n_max, const float* scores,
                                const int32_t* lengths, const int32_t* keep_counts,
                                const int32_t* keep_idx, int32_t max_keep,
                                const int32_t* evict_idx, int32_t max_evict);
dropkv_status run_select(int32_t B, int32_t Hkv, int32_t n_max, const float* scores,
                         const int32_t* lengths, const int32_t* keep_counts, int32_t* keep_idx,
                         int32_t max_keep, int32_t* evict_idx, int32_t max_evict,
                         int32_t* status_word, cudaStream_t st);
dropkv_status cuda_fail(cudaError_t e);

}  // namespace dropkv
