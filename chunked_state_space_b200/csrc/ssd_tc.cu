// Tensor-core kernels of libssd (tcgen05 / TMEM / TMA, sm_100a): the fused
// kernel (ssd_fused.cu) serves the whole scan and, in its per-chunk modes,
// steps 2 and 4; nothing else needs workspace.
#include "ssd_tc.cuh"

namespace ssd {

size_t tc_workspace_bytes(const Problem&) { return 0; }

}  // namespace ssd
