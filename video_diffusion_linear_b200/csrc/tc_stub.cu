// Placeholder launchers of the tensor-core path until its kernels land.
#include "internal.h"
namespace vdn {
cudaError_t launch_stats_tc(const Args&, float*, uint32_t*) { return cudaErrorNotSupported; }
cudaError_t launch_scan_tc(const Args&, const float*, const uint16_t*, float*, float*, bool, uint32_t*) {
  return cudaErrorNotSupported;
}
cudaError_t launch_readout_tc(const Args&, const uint16_t*, uint32_t*) { return cudaErrorNotSupported; }
}  // namespace vdn
