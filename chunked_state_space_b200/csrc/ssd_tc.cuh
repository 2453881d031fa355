// Tensor-core (tcgen05 / TMEM / TMA) kernels of libssd: declarations.
#pragma once

#include "ssd_common.cuh"

namespace ssd {

// True when the tcgen05 step kernels cover this problem (bf16 io and the
// tile sizes they are written for).
bool tc_supported(const Problem& p);
// True when a fused single-pass kernel covers this problem (the one-head
// kernel always does; the two-head kernel when pair_supported also holds).
bool fused_supported(const Problem& p);
// True when the two-heads-per-CTA kernel covers it (even heads per group).
bool pair_supported(const Problem& p);
// True when launch_fused runs the two-head kernel for this problem.
bool uses_pair_kernel(const Problem& p);
// Kernel launches of one fused call.
int fused_kernels_per_call(const Problem& p);
// Workspace bytes the tensor-core paths need (0 if unsupported): the two-head
// kernel's carries between CTAs when it splits sequences across them.
size_t tc_workspace_bytes(const Problem& p);
size_t pair_workspace_bytes(const Problem& p);

cudaError_t launch_chunk_scan_tc(const Problem& p, const float* lam, const float* prev, cudaStream_t st);
// Segments per sequence of the two-head kernel's schedule: 0 = chosen from
// the shape (the default), n > 0 = n wherever n divides the sub-chunks
// (self-tests of the carries).
void set_pair_segments(int nseg);
// Segments per sequence of the one-head kernel's segmented form (problems
// with fewer sequences than SMs, or the last partial round of sequences):
// 0 = chosen by its cost model, n > 0 = about n segments whatever the size,
// with the first `whole` sequences run whole (self-tests).
void set_fused_segments(int nseg);
void set_fused_split(int nseg, int64_t whole);
cudaError_t launch_segment_states(const Problem& p, int64_t whole, float* states, float* seg_decay,
                                  cudaStream_t st);
cudaError_t launch_segment_scan(const Problem& p, int64_t whole, const float* prev, const float* init,
                                float* final_state, cudaStream_t st);
// Step 2 on tensor cores: every chunk's end state from a zero start, several
// consecutive chunks of one (batch, head) per CTA (csrc/ssd_lean.cu).
cudaError_t launch_chunk_states_seq(const Problem& p, const float* lam, float* states, cudaStream_t st);
// Consecutive chunks per CTA of the tensor-core step kernels (steps 2 and 4),
// and its self-test override (n > 0: n chunks per CTA; 0: from the shape).
int64_t step_chunks_per_cta(const Problem& p);
void set_step_chunks_per_cta(int n);
// The whole scan in one launch.  With a workspace of pair_workspace_bytes
// the two-head kernel runs segments of the sequences round-robin on one
// persistent CTA per SM; without one (NULL / too small) every CTA runs whole
// sequences.
cudaError_t launch_fused(const Problem& p, const float* init, float* final_state, void* workspace,
                         size_t workspace_bytes, cudaStream_t st);
// The RMS norm between the layers of a stack, fused into the one-head kernel:
// ss_in holds, per (batch, token, head), the sum of squares of the input row
// (the previous layer's stored y), from which each token's scale
// r_t = 1 / sqrt(sum_h ss_in / (H P) + eps) is applied on the fly; ss_out
// receives the same sums for this call's stored y.  Both [B][L][H] f32 with
// token stride H and batch stride batch_stride; either may be NULL.
struct NormIO {
  const float* ss_in;
  float* ss_out;
  int64_t batch_stride;
  float eps;
};
cudaError_t launch_fused_normed(const Problem& p, const float* init, float* final_state, const NormIO& norm,
                                cudaStream_t st);
// withhold: 0 normal; 1 no TMA loads; 2 no carries published (self-tests of the bounded waits)
cudaError_t launch_pair(const Problem& p, const float* init, float* final_state, void* workspace,
                        size_t workspace_bytes, cudaStream_t st, int withhold);

}  // namespace ssd
