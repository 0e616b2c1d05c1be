// selftest.cu -- device-side checks of the bounded waits the tensor-core and
// select kernels rely on, with no fault, trap or unbounded spin involved:
//   dropkv_selftest_wait_timeout: one CTA waits on an mbarrier that nothing
//     ever arrives on, with the same bounded wait (a %globaltimer limit) those
//     kernels use, and reports DROPKV_ERR_TIMEOUT in the caller's status word
//     when the wait gives up;
//   dropkv_selftest_select_timeout: the select kernel itself, with one CTA of
//     every cluster withholding an arrival and a short wait limit, so that the
//     caller sees the timeout status and keep / evict lists of -1.
// The kernels return and the context stays usable.
#include "internal.h"
#include "tc_ptx.cuh"

namespace dropkv {
namespace {

__global__ void k_wait_timeout(int32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = tc::smem_u32(&bar);
  if (threadIdx.x == 0) {
    tc::mbar_init(b, 1);
    tc::fence_mbar_init();
  }
  __syncthreads();
  // phase 0 never completes: no thread arrives
  if (threadIdx.x == 0 && !tc::mbar_wait(b, 0, limit_ns)) atomicMax(status, (int)DROPKV_ERR_TIMEOUT);
}

}  // namespace
}  // namespace dropkv

extern "C" {

dropkv_status dropkv_selftest_wait_timeout(int32_t* status_dev, uint64_t limit_ns, void* stream) {
  if (!status_dev || ((uintptr_t)status_dev & 3u) || limit_ns == 0 || limit_ns > 1000000000ull)
    return DROPKV_ERR_ARG;
  const dropkv_status r = dropkv::device_ok();
  if (r != DROPKV_OK) return r;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  dropkv::k_wait_timeout<<<1, 32, 0, st>>>(status_dev, limit_ns);
  return cudaGetLastError() == cudaSuccess ? DROPKV_OK : DROPKV_ERR_CUDA;
}

dropkv_status dropkv_selftest_select_timeout(int32_t B, int32_t Hkv, int32_t n_max,
                                             const float* scores, const int32_t* lengths,
                                             const int32_t* keep_counts, int32_t* keep_idx,
                                             int32_t max_keep, int32_t* evict_idx,
                                             int32_t max_evict, int32_t* status_dev,
                                             uint64_t limit_ns, void* stream) {
  dropkv_status r = dropkv::check_select_args(B, Hkv, n_max, scores, lengths, keep_counts,
                                              keep_idx, max_keep, evict_idx, max_evict);
  if (r != DROPKV_OK) return r;
  if (B > dropkv::kMaxB || !status_dev || ((uintptr_t)status_dev & 3u) || limit_ns == 0 ||
      limit_ns > 1000000000ull)
    return DROPKV_ERR_ARG;
  r = dropkv::device_ok();
  if (r != DROPKV_OK) return r;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaError_t e = cudaMemsetAsync(status_dev, 0, sizeof(int32_t), st))
    return dropkv::cuda_fail(e);
  int32_t L[dropkv::kMaxB], K[dropkv::kMaxB];
  for (int b = 0; b < B; ++b) {
    L[b] = lengths ? lengths[b] : n_max;
    K[b] = keep_counts[b];
  }
  if (cudaError_t e = dropkv::launch_select_stalled(B, Hkv, n_max, scores, L, K, keep_idx,
                                                   max_keep, evict_idx, max_evict, status_dev,
                                                   limit_ns, st))
    return dropkv::cuda_fail(e);
  return DROPKV_OK;
}

}  // extern "C"
