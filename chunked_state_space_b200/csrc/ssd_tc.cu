// Tensor-core kernels of libssd (tcgen05 / TMEM / TMA, sm_100a).
#include "ssd_tc.cuh"

namespace ssd {

bool tc_supported(const Problem&) { return false; }
size_t tc_workspace_bytes(const Problem&) { return 0; }

cudaError_t launch_chunk_state_tc(const Problem&, const float*, float*, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_chunk_scan_tc(const Problem&, const float*, const float*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace ssd
