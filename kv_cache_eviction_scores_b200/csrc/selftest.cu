// selftest.cu -- a device-side check of the bounded waits the tensor-core and
// select kernels rely on: one CTA waits on an mbarrier that nothing ever
// arrives on, with the same bounded wait (a %globaltimer limit) those kernels
// use, and reports DROPKV_ERR_TIMEOUT in the caller's status word when the
// wait gives up.  No fault, trap or unbounded spin is involved: the kernel
// returns and the context stays usable.
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

}  // extern "C"
