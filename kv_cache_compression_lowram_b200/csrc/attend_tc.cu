// Steps 3-5 on tcgen05 tensor cores (placeholder until the kernel lands).
#include "lowram_internal.cuh"

namespace lowram {

bool attend_tc_supported(const Geom&, int, int) { return false; }

cudaError_t launch_attend_tc(const Geom&, const CacheBuffers&, const Scratch&, int, const void*,
                             int, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace lowram
