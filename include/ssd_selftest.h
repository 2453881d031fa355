/*
 * ssd_selftest.h -- diagnostic entry point of libssd.so (no counterpart on the
 * pages: it checks the tensor-core building blocks the scan kernels are made
 * of, not the scan).
 *
 * ssd_selftest_umma computes D[128 x N] = A[128 x K] * B[K x N] on one CTA
 * with bf16 inputs and fp32 accumulation through tcgen05.mma, staging the
 * operands in the layout named by `variant`:
 *   SSD_SELFTEST_A_K_B_K            A [128][K] and B [N][K] in global, both K-major in smem
 *   SSD_SELFTEST_A_K_B_MN           A [128][K] K-major, B [K][N] MN-major
 *   SSD_SELFTEST_A_MN_B_MN          A [K][128] MN-major, B [K][N] MN-major
 *   SSD_SELFTEST_A_MN_B_MN_SWAPPED  as above with the two descriptor strides exchanged
 *                                   (expected to be wrong; documents the encoding)
 *   SSD_SELFTEST_TS_A_TMEM_B_MN     A [128][K] placed in tensor memory, B [K][N] MN-major
 *   SSD_SELFTEST_TMA_A_K_B_MN       as A_K_B_MN but both operands loaded by TMA
 * A, B: device bf16, D: device fp32 [128][N]; N in {64, 128}; K in {64, 128, 256};
 * 16-byte aligned.  Asynchronous on `stream`.  Errors: SSD_ERR_INVALID_ARG,
 * SSD_ERR_UNSUPPORTED, SSD_ERR_ALIGN, SSD_ERR_CUDA; a bounded wait that gives
 * up raises the status read by ssd_read_device_status.
 */
#ifndef SSD_B200_SSD_SELFTEST_H
#define SSD_B200_SSD_SELFTEST_H

#include "ssd.h"

#ifdef __cplusplus
extern "C" {
#endif

enum {
  SSD_SELFTEST_A_K_B_K = 0,
  SSD_SELFTEST_A_K_B_MN = 1,
  SSD_SELFTEST_A_MN_B_MN = 2,
  SSD_SELFTEST_A_MN_B_MN_SWAPPED = 3,
  SSD_SELFTEST_TS_A_TMEM_B_MN = 4,
  SSD_SELFTEST_TMA_A_K_B_MN = 5
};

ssd_status ssd_selftest_umma(int32_t variant, const void* A, const void* B, float* D, int32_t N, int32_t K,
                             void* stream);

/*
 * ssd_selftest_fused_trace runs ssd_scan_fwd's fused tensor-core kernel (same
 * arguments; the problem must be one the fused kernel takes, else
 * SSD_ERR_UNSUPPORTED) and has the CTA of batch 0, head 0 write the SM clock
 * (clock64) of each pipeline event of each 128-token sub-chunk j to
 * trace[24*j + e] (device buffer of trace_len >= 24*ceil(L/128) uint64):
 * e = 0 loads issued, 1 S issued, 2 products issued, 3 mask started, 4 mask
 * done, 5 lam ready, 6 X' done, 7 products seen by the epilogue, 8 state
 * published, 9 epilogue done, 10 products ready to issue, 11 first third of
 * the products issued, 12 S ready to issue, 13-17 points inside the mask
 * (first TMEM read, blocks 0-1 written, second read, blocks 2-3 written,
 * stores complete).  After those 24*ceil(L/128) values, every CTA c (batch
 * b, head h: c = b*H + h) writes trace[24*ceil(L/128) + 3c + {0, 1, 2}] =
 * its start and end (globaltimer, ns) and its SM index; trace_len must cover
 * them.  Used to find the critical path and the spread of CTA durations.
 */
ssd_status ssd_selftest_fused_trace(const ssd_dims* d, const void* x, const float* dt, const float* A,
                                    const void* Bm, const void* Cm, const float* D, const float* init_state,
                                    void* y, float* final_state, unsigned long long* trace, int64_t trace_len,
                                    void* stream);

/*
 * ssd_selftest_timeout exercises the bounded waits of ssd_scan_fwd's fused
 * tensor-core kernel (the two-head kernel when d->flags has
 * SSD_FLAG_TWO_HEADS_PER_CTA and it takes the shape, else the one-head kernel): same
 * arguments and validation as ssd_scan_fwd (the problem must be one a fused
 * kernel takes, else SSD_ERR_UNSUPPORTED), but
 * the kernel issues none of its TMA loads, so every wait on them gives up
 * after about one second.  The launch itself returns SSD_OK; the following
 * ssd_read_device_status(stream) must return SSD_ERR_TIMEOUT (and clears the
 * word).  y and final_state are left undefined.  No fault, trap or unbounded
 * wait is involved: the kernel drains and exits, and later launches in the
 * same context run normally.
 */
ssd_status ssd_selftest_timeout(const ssd_dims* d, const void* x, const float* dt, const float* A, const void* Bm,
                                const void* Cm, const float* D, const float* init_state, void* y, float* final_state,
                                void* stream);

/*
 * ssd_selftest_carry_timeout exercises the one wait of the two-head fused
 * kernel that is not on a barrier of its own CTA: in its segmented schedule a
 * segment after the first waits for the CTA that ran the segment before it to
 * publish that sequence's state (the page's inter-chunk recursion, "分块推理…"
 * §2.2, handed across CTAs).  Same arguments and validation as ssd_scan_fwd
 * plus the workspace; d->flags must request the two-head kernel
 * (SSD_FLAG_TWO_HEADS_PER_CTA) and the problem be one it segments (even heads
 * per group, and more than one segment per sequence, chosen from the shape or
 * set by ssd_selftest_set_segments), else SSD_ERR_UNSUPPORTED.  No
 * carry is ever published, so those waits give up after about two seconds;
 * the launch returns SSD_OK and the following ssd_read_device_status(stream)
 * returns SSD_ERR_TIMEOUT.  y and final_state are left undefined; nothing
 * faults and the context stays usable.
 */
ssd_status ssd_selftest_carry_timeout(const ssd_dims* d, const void* x, const float* dt, const float* A,
                                      const void* Bm, const void* Cm, const float* D, const float* init_state,
                                      void* y, float* final_state, void* workspace, size_t workspace_bytes,
                                      void* stream);

/*
 * ssd_selftest_set_segments sets how many segments the two-head kernel cuts
 * each sequence into for the following launches of this process (host state,
 * not thread-safe): nseg > 0 wherever nseg divides the sequence's 128-token
 * sub-chunks (else whole sequences), 0 = chosen from the shape (the default).
 * It also forces the one-head kernel's segmented form (three launches: the
 * segments' end states, their combine, the segments' scans) with about nseg
 * segments of whole sub-chunks, whatever the problem's size.
 * With fewer head pairs than SMs a forced segmentation puts a segment and its
 * predecessor in the same round, so the later one waits for the earlier one:
 * correct, slower.  Returns SSD_ERR_INVALID_ARG for nseg < 0.
 */
ssd_status ssd_selftest_set_segments(int nseg);

/*
 * ssd_selftest_set_split forces the one-head kernel's segmented form for the
 * following launches of this process (host state, not thread-safe), in its
 * mixed layout: the first `whole` (batch, head) sequences (in batch-major
 * order) are scanned whole by one CTA each, from the caller's initial state
 * to its final state, and every later sequence is cut into about nseg
 * segments of whole 128-token sub-chunks (end states, combine, segment
 * scans).  whole is clamped to B*H - 1; nseg = 0 restores the cost model's
 * choice (which uses this layout when B*H exceeds a whole number of rounds
 * of CTAs on the SMs by a partial round).  The two-head kernel is not
 * affected.  Returns SSD_ERR_INVALID_ARG for nseg < 0 or whole < 0.
 * Same arithmetic as the default path: results equal one CTA per sequence
 * up to the rounding of the segments' combine.
 */
ssd_status ssd_selftest_set_split(int nseg, int64_t whole);

/*
 * ssd_selftest_set_step_chunks sets how many consecutive chunks of one
 * (batch, head) sequence each CTA of the tensor-core step kernels handles
 * (ssd_chunk_state and ssd_chunk_scan, and the step-by-step scan) for the
 * following launches of this process (host state, not thread-safe): n > 0
 * forces n (at most the chunks of a sequence), 0 restores the choice from the
 * shape.  Same results either way.  Returns SSD_ERR_INVALID_ARG for n < 0.
 */
ssd_status ssd_selftest_set_step_chunks(int n);

#ifdef __cplusplus
}
#endif

#endif /* SSD_B200_SSD_SELFTEST_H */
