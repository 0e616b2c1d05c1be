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
// race.  The only part of the scratch that must start at zero is the 4-byte
// status word of the select kernels: each call enqueues one cudaMemsetAsync of
// it on the caller's stream before its kernels.  That word is not returned to
// the caller: a select kernel whose bounded wait gives up fills the lists of
// its (b, h) with -1 instead.
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
  NvtxRange range("dropkv_select_noalloc");
  dropkv_status r = check_select_args(B, Hkv, n_max, scores, lengths, keep_counts, keep_idx,
                                      max_keep, evict_idx, max_evict);
  if (r != DROPKV_OK) return r;
  // the scratch a launch slice needs must fit the static array
  const int Bs = B < kMaxB ? B : kMaxB;
  if (select_workspace_bytes(Bs, Hkv, n_max) > kNoAllocScratchBytes) return DROPKV_ERR_WORKSPACE;
  r = device_ok();
  if (r != DROPKV_OK) return r;
  void* ws = nullptr;
  if (cudaError_t e = scratch_ptr(&ws)) return cuda_fail(e);
  return run_select(B, Hkv, n_max, scores, lengths, keep_counts, keep_idx, max_keep, evict_idx,
                    max_evict, reinterpret_cast<int32_t*>(ws),
                    reinterpret_cast<cudaStream_t>(stream));
}
