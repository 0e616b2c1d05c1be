// tc.cu -- tensor-core (tcgen05 + TMA) scoring path.
#include "internal.h"

namespace dropkv {

bool tc_available() { return false; }
int tc_split_target() { return 296; }
int tc_launch_count() { return 3; }

cudaError_t launch_tc_scores(const dropkv_shape&, const void*, const void*, const void*,
                             const Lens&, const ScoresLayout&, char*, float*, float*, int32_t*,
                             cudaStream_t, KernelEvents&) {
  return cudaErrorNotSupported;
}

}  // namespace dropkv
