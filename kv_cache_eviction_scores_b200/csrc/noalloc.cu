// noalloc.cu -- dropkv_select_noalloc: the eviction step for callers that
// cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: for example code that runs inside a
// serving engine which owns all device memory through its own pool and refuses
// any other allocation, or a latency-critical path where the implicit device
// synchronisation of cudaMalloc is not acceptable.  Such a caller cannot supply
// the workspace dropkv_select asks for.  This entry point runs the same select
// kernels on a scratch array that is compiled into the library instead.
//
// The scratch lives in static device memory: every GPU that loads the library
// holds these bytes until the process exits.  The first call on a device looks
// up the array's device address with cudaGetSymbolAddress (with that device
// current) and caches it; because that lookup is a runtime call, the first call
// on each device should happen before any stream capture.  All calls share the
// one array, so calls whose work overlaps on the GPU (on different streams)
// race; the kernels themselves reset every part of the scratch that must start
// at zero at the beginning of each call.
#include <mutex>

#include "internal.h"

namespace dropkv {
namespace {

// Scratch of the select kernels here: 4 KiB (the select path keeps its state
// in shared memory and needs only a status word, for any size).
constexpr size_t kNoAllocScratchBytes = size_t(4) << 10;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_select_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_select_scratch on the current device (looked up once per
// device; the host-side name of the array is not a device address).
cudaError_t scratch_ptr(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_select_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace dropkv

using namespace dropkv;

extern "C" dropkv_status dropkv_select_noalloc(int32_t B, int32_t Hkv, int32_t n_max,
                                               const float* scores, const int32_t* lengths,
                                               const int32_t* keep_counts, int32_t* keep_idx,
                                               int32_t max_keep, int32_t* evict_idx,
                                               int32_t max_evict, void* stream) {
  if (B < 1 || Hkv < 1 || n_max < 1 || !scores || !keep_counts) return DROPKV_ERR_ARG;
  if ((!keep_idx && max_keep > 0) || (!evict_idx && max_evict > 0)) return DROPKV_ERR_ARG;
  if (max_keep < 0 || max_evict < 0) return DROPKV_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(scores) & 15u) || (reinterpret_cast<uintptr_t>(keep_idx) & 3u) ||
      (reinterpret_cast<uintptr_t>(evict_idx) & 3u))
    return DROPKV_ERR_ARG;
  if ((double)B * Hkv * (double)n_max > 4.0e18) return DROPKV_ERR_ARG;
  for (int b = 0; b < B; ++b) {
    const int L = lengths ? lengths[b] : n_max;
    if (L < 0 || L > n_max) return DROPKV_ERR_ARG;
    if (keep_counts[b] < 0 || keep_counts[b] > L) return DROPKV_ERR_ARG;
    if (keep_counts[b] > max_keep || L - keep_counts[b] > max_evict) return DROPKV_ERR_ARG;
  }
  // the scratch a launch slice needs must fit the static array
  const int Bs = B < kMaxB ? B : kMaxB;
  if (select_workspace_bytes(Bs, Hkv, n_max) > kNoAllocScratchBytes) return DROPKV_ERR_WORKSPACE;
  int dev = -1, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    cudaGetLastError();
    return DROPKV_ERR_UNSUPPORTED;
  }
  if (major != 10) return DROPKV_ERR_UNSUPPORTED;
  void* ws = nullptr;
  if (scratch_ptr(&ws) != cudaSuccess) return DROPKV_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  for (int b0 = 0; b0 < B; b0 += kMaxB) {
    const int n = (B - b0) < kMaxB ? (B - b0) : kMaxB;
    int32_t L[kMaxB], K[kMaxB];
    for (int i = 0; i < n; ++i) {
      L[i] = lengths ? lengths[b0 + i] : n_max;
      K[i] = keep_counts[b0 + i];
    }
    const size_t seg0 = (size_t)b0 * Hkv;
    if (launch_select(n, Hkv, n_max, scores + seg0 * n_max, L, K, keep_idx + seg0 * max_keep,
                      max_keep, evict_idx + seg0 * max_evict, max_evict, ws, st) != cudaSuccess)
      return DROPKV_ERR_CUDA;
  }
  return DROPKV_OK;
}
