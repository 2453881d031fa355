// Tensor-core (tcgen05 / TMEM / TMA) kernels of libssd: declarations.
#pragma once

#include "ssd_common.cuh"

namespace ssd {

// True when the tcgen05 step kernels cover this problem (bf16 io and the
// tile sizes they are written for).
bool tc_supported(const Problem& p);
// True when the fused single-pass kernel covers this problem.
bool fused_supported(const Problem& p);
// Kernel launches of one fused call.
int fused_kernels_per_call(const Problem& p);
// Workspace bytes the tensor-core paths need (0 if unsupported).
size_t tc_workspace_bytes(const Problem& p);

cudaError_t launch_chunk_state_tc(const Problem& p, const float* lam, float* states, cudaStream_t st);
cudaError_t launch_chunk_scan_tc(const Problem& p, const float* lam, const float* prev, cudaStream_t st);
cudaError_t launch_fused(const Problem& p, const float* init, float* final_state, void* workspace,
                         cudaStream_t st);

}  // namespace ssd
