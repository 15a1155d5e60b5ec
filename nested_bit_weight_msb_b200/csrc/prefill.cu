// Prefill path (M > 16): placeholder until the tcgen05 kernel lands.
#include "common.cuh"
#include "internal.h"

namespace matq {

size_t prefill_workspace_bytes(int M, int K, int group) {
  (void)group;
  return (((size_t)M * K * 2) + 255) & ~size_t(255);
}

cudaError_t launch_prefill(const void*, int, int, const void*, const PlaneGeom&, const uint16_t*, const uint8_t*, int,
                           int, void*, int, void*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace matq
