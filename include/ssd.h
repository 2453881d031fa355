/*
 * ssd.h -- C ABI of the B200 chunked selective-state-space (SSD) scan library
 *          (libssd.so, sm_100a).
 *
 * What it computes.  For every batch b and head h, with group g = h / (H/G):
 *     a_t = exp(dt[b,t,h] * A[h])
 *     h_t = a_t h_{t-1} + B[b,t,g,:] x[b,t,h,:]^T          (N x P state)
 *     y_t = C[b,t,g,:]^T h_t + D[h] x[b,t,h,:]
 * starting from init_state (or zero).  This is the recurrence of
 * "分块推理：解锁循环模型并行计算，实现长序列高效处理" §2, with the per-token (selective)
 * dt, B, C of "告别Transformer的二次方噩梦：用Mamba（S6）模型在长文本任务中实现线性时间推理"
 * §2.1.  The library evaluates it chunk by chunk as that page's §2.1-§2.2
 * derive: chunks of Q tokens, (1) a cumulative sum of the log-decays
 * dt*A inside each chunk, (2) the chunk-local state b_intra(c) from a zero
 * start, (3) the inter-chunk recursion b(c) = b_intra(c) + (prod a) b(c-1),
 * and (4) the outputs by_intra (masked C B^T (.) L times X) plus the
 * correction by_inter = diag(L) C(c) b(c-1).  ssd_vertical_fwd adds the
 * page's §3.2 depth-first multi-layer schedule.
 *
 * Conventions shared by every entry point.
 *  - Ownership: the caller allocates and owns every buffer.  The library
 *    never allocates device memory and never synchronises the stream.
 *  - Pointers: device pointers unless stated; each must be 16-byte aligned.
 *  - Layout: contiguous row-major tensors:
 *        x, y    [B, L, H, P]   (io dtype)      dt [B, L, H] (f32)
 *        Bm, Cm  [B, L, G, N]   (io dtype)      A, D [H] (f32)
 *        states  [B, H, N, P]   (f32)
 *        lam     [B, H, nc, Q]  (f32), nc = ceil(L / Q)
 *        chunk states / prev states [B, H, nc, N, P] (f32)
 *  - dt must be positive and A non-positive (no softplus, bias or clamp is
 *    applied); results for dt*A > 0 may overflow.
 *  - L need not be a multiple of Q: the last chunk may be shorter.
 *  - Streams: `stream` is a cudaStream_t (NULL = legacy default stream);
 *    work is enqueued asynchronously on it.
 *  - Errors: a status other than SSD_OK means no kernel was launched, except
 *    SSD_ERR_CUDA (a launch failed part-way) and SSD_ERR_TIMEOUT (reported by
 *    ssd_read_device_status after a bounded device-side wait gave up).
 *  - Results are deterministic run to run (no atomics in reductions).
 *  - Per-device set-up: on its first call on a device the library records a
 *    few things it keeps for the life of the process (the kernels' shared-
 *    memory opt-in, the built-in scratch buffer's device address, the streams
 *    and events of the wavefront and host-copy schedules).  Resetting the
 *    device (cudaDeviceReset) after that first call is not supported: the
 *    recorded state would belong to the destroyed context.
 */
#ifndef SSD_B200_SSD_H
#define SSD_B200_SSD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SSD_OK = 0,
  SSD_ERR_INVALID_ARG = 1, /* NULL where a pointer is required, bad enum, aliasing */
  SSD_ERR_SHAPE = 2,       /* non-positive size, H % G != 0 */
  SSD_ERR_DTYPE = 3,       /* io dtype not supported for this call */
  SSD_ERR_ALIGN = 4,       /* pointer not 16-byte aligned */
  SSD_ERR_UNSUPPORTED = 5, /* size outside the supported set (see ssd_dims) */
  SSD_ERR_WORKSPACE = 6,   /* workspace NULL or smaller than the size query */
  SSD_ERR_CUDA = 7,        /* a CUDA launch or query failed */
  SSD_ERR_TIMEOUT = 8      /* a bounded device-side wait gave up */
} ssd_status;

typedef enum { SSD_F32 = 0, SSD_BF16 = 1 } ssd_dtype;

/*
 * Problem sizes.  Supported: batch, seqlen >= 1; 1 <= headdim (P) <= 64;
 * 1 <= dstate (N) <= 128; 1 <= chunk (Q) <= 256; ngroups >= 1 dividing nheads.
 * io_dtype is the dtype of x, Bm, Cm and y.  flags: a combination of
 * ssd_flags (any other bit is SSD_ERR_INVALID_ARG).
 */
typedef struct ssd_dims {
  int64_t batch;    /* B */
  int64_t seqlen;   /* L */
  int64_t nheads;   /* H */
  int64_t headdim;  /* P */
  int64_t dstate;   /* N */
  int64_t ngroups;  /* G */
  int64_t chunk;    /* Q */
  int32_t io_dtype; /* ssd_dtype */
  int32_t flags;    /* ssd_flags */
} ssd_dims;

/*
 * SSD_FLAG_INPUT_DT: the input enters scaled by dt, h_t = a_t h_{t-1} +
 * dt_t B_t x_t^T (the discretisation of the selective-scan page: the
 * input-dependent step Delta scales the input term as well as the decay);
 * the skip stays D_h x_t with the unscaled x.  Taken by ssd_scan_fwd,
 * ssd_scan_fwd_strided, ssd_scan_fwd_host and ssd_vertical_fwd when the
 * tensor-core path takes the shape, and by ssd_step; every other entry point
 * (and ssd_scan_fwd on the CUDA-core path) returns SSD_ERR_UNSUPPORTED.
 *
 * SSD_FLAG_TWO_HEADS_PER_CTA: run the fused scan with two heads of a group per
 * CTA (they share their B and C tiles, S = C B^T and the state products) where
 * the shape allows it (an even number of heads per group); same results within
 * rounding.  Kept for comparison: on B200 it measured slower than the default
 * one-head kernel (its per-row CUDA-core work has half the warps per head).
 * Changes nothing on other paths.
 */
typedef enum { SSD_FLAG_INPUT_DT = 1, SSD_FLAG_TWO_HEADS_PER_CTA = 2 } ssd_flags;

/* Human-readable name of a status code (static string, never NULL). */
const char* ssd_status_string(ssd_status s);

/* Library version as 10000*major + 100*minor + patch. */
int ssd_version(void);

/*
 * Bytes of device workspace ssd_scan_fwd needs for `d` (written to *bytes).
 * Errors: SSD_ERR_INVALID_ARG (NULL), SSD_ERR_SHAPE, SSD_ERR_UNSUPPORTED,
 * SSD_ERR_DTYPE.
 */
ssd_status ssd_scan_workspace_size(const ssd_dims* d, size_t* bytes);

/*
 * One layer of the chunked scan, "分块推理…" §2.1-§2.2: y and the final state
 * from x, dt, A, Bm, Cm, D and the initial state, all four steps on `stream`.
 *   x [B,L,H,P] io, dt [B,L,H] f32, A [H] f32, Bm/Cm [B,L,G,N] io,
 *   D [H] f32 or NULL (= 0), init_state [B,H,N,P] f32 or NULL (= 0),
 *   y [B,L,H,P] io (written; must not overlap any input),
 *   final_state [B,H,N,P] f32 or NULL (may alias init_state),
 *   workspace: device scratch of at least ssd_scan_workspace_size bytes,
 *   owned by the caller, contents need not be initialised.
 * Picks the tensor-core path for bf16 io when the sizes allow it, else the
 * CUDA-core path (ssd_scan_path says which, and how many launches).
 * Errors: every status above.
 */
ssd_status ssd_scan_fwd(const ssd_dims* d, const void* x, const float* dt, const float* A,
                        const void* Bm, const void* Cm, const float* D, const float* init_state,
                        void* y, float* final_state, void* workspace, size_t workspace_bytes,
                        void* stream);

/*
 * ssd_scan_fwd on strided tensors (tensor-core path only: bf16 io, P = 64,
 * N = 128, Q a multiple of 128; else SSD_ERR_UNSUPPORTED), e.g. x, B and C as
 * column slices of one fused projection output [B, L, H*P + 2*G*N].  Each of
 * x, dt, Bm/Cm (one stride pair for both) and y takes a batch stride and a
 * token stride in ELEMENTS; inside a token the heads (groups) stay dense:
 *   x[b, t, h, p]  at x  + b*x_bstride  + t*x_tstride  + h*P + p
 *   dt[b, t, h]    at dt + b*dt_bstride + t*dt_tstride + h
 *   Bm[b, t, g, n] at Bm + b*bc_bstride + t*bc_tstride + g*N + n (Cm alike)
 *   y like x with y_bstride, y_tstride.
 * A, D, init_state, final_state are contiguous as in ssd_scan_fwd.  Token
 * strides must be at least the dense row (H*P, H, G*N), batch strides at
 * least a whole sequence (else SSD_ERR_SHAPE); the bf16 strides must be
 * multiples of 8 elements (TMA: 16 bytes) and the pointers 16-byte aligned
 * (dt: 4 bytes) (else SSD_ERR_ALIGN); y must not overlap x, dt, Bm or Cm
 * (SSD_ERR_INVALID_ARG).  No workspace is needed.
 */
ssd_status ssd_scan_fwd_strided(const ssd_dims* d, const void* x, int64_t x_bstride, int64_t x_tstride,
                                const float* dt, int64_t dt_bstride, int64_t dt_tstride, const float* A,
                                const void* Bm, const void* Cm, int64_t bc_bstride, int64_t bc_tstride,
                                const float* D, const float* init_state, void* y, int64_t y_bstride,
                                int64_t y_tstride, float* final_state, void* stream);

/*
 * Bytes of DEVICE workspace ssd_scan_fwd_host needs for `d`: A and D, and two
 * slice buffers (one sequence, up to 4096 tokens: inputs, outputs, the end
 * state and the scan's scratch).
 */
ssd_status ssd_scan_fwd_host_workspace_size(const ssd_dims* d, size_t* bytes);

/*
 * ssd_scan_fwd with every tensor in HOST memory (same shapes, layouts and
 * meaning; init_state, final_state and D may be NULL as there), the copies
 * overlapped with the scan: the batch flows through the device workspace in
 * slices of one sequence and up to 4096 tokens (a whole number of chunks),
 * slice s+1 copied in and slice s-1 copied out while slice s is scanned on
 * `stream`, each slice from the end state of the slice before it in its
 * sequence (the chunk recursion of "分块推理…" §2.2 with the slice as the chunk).
 * Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister):
 * pageable memory works but its copies do not overlap.  The host buffers must
 * stay valid and unchanged until the work on `stream` completes; y and
 * final_state are written by then.  Results equal ssd_scan_fwd's up to
 * rounding (bitwise when the sequence is one slice and both choose the same
 * split of the sequences over SMs).  The two copy streams and their events belong to the
 * library (one set per device, created on first use, kept until the process
 * exits); each call forks them from `stream` and joins them back.  Calls from
 * several host threads on one device are serialised while they enqueue.
 * Errors: as ssd_scan_fwd; SSD_ERR_WORKSPACE if the device workspace is NULL
 * or smaller than ssd_scan_fwd_host_workspace_size.
 */
ssd_status ssd_scan_fwd_host(const ssd_dims* d, const void* x, const float* dt, const float* A, const void* Bm,
                             const void* Cm, const float* D, const float* init_state, void* y, float* final_state,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * Which implementation ssd_scan_fwd uses for `d`: *path = SSD_PATH_CUDA_CORES
 * (four CUDA-core step kernels), SSD_PATH_TENSOR_STEPS (four step kernels,
 * steps 2 and 4 on tcgen05 tensor cores), SSD_PATH_FUSED (one tensor-core
 * kernel) or SSD_PATH_FUSED_PAIR (one tensor-core kernel, two heads of a
 * group per CTA sharing their B and C tiles; SSD_FLAG_TWO_HEADS_PER_CTA).
 * The one-head kernel runs one (batch, head) sequence per CTA; where that
 * leaves SMs idle (fewer sequences than SMs, or B*H a whole number of rounds
 * of CTAs on the SMs plus a partial round) and a cost model of CTA rounds
 * predicts a gain, it runs the segmented form instead (three launches: the
 * end state of every segment of the affected sequences from a zero start,
 * their ordered combine, then one grid scanning the other sequences whole and
 * every segment from its start state), which needs the workspace of
 * ssd_scan_workspace_size (without it, whole sequences).  The two-head
 * kernel, given that workspace and more head pairs than SMs, cuts every
 * sequence into segments scheduled in rounds on one persistent CTA per SM and
 * hands the state across segment boundaries through the workspace; otherwise
 * it runs whole sequences;
 * *kernels = kernel launches per call.  Either output pointer may be NULL.
 * Errors: as ssd_scan_workspace_size.
 */
enum { SSD_PATH_CUDA_CORES = 0, SSD_PATH_TENSOR_STEPS = 1, SSD_PATH_FUSED = 2, SSD_PATH_FUSED_PAIR = 3 };
ssd_status ssd_scan_path(const ssd_dims* d, int32_t* path, int32_t* kernels);

/* The same computation, forced through the four separate step kernels below
 * (the step-testable path).  Same arguments and errors as ssd_scan_fwd. */
ssd_status ssd_scan_fwd_unfused(const ssd_dims* d, const void* x, const float* dt, const float* A,
                                const void* Bm, const void* Cm, const float* D,
                                const float* init_state, void* y, float* final_state,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * The step-by-step scan (same arguments, results and errors as
 * ssd_scan_fwd_unfused) for callers that cannot allocate device memory when
 * they run it -- code being captured into a CUDA graph, engines or plugin
 * hosts that plan all device memory up front, runtimes with a fixed budget.
 * The pages have no counterpart: this is a packaging of the same kernels.
 *   - Scratch comes from a 32 MiB buffer compiled into libssd (every GPU that
 *     loads the library holds it until the process exits).  The call needs
 *     4*B*H*nc*Q + 4*B*H*nc*N*P bytes (each part rounded up to 256) and returns
 *     SSD_ERR_UNSUPPORTED, with a message on stderr, for sizes beyond that.
 *   - The call allocates nothing (no cudaMalloc or cudaFree, no allocating
 *     library routine).  Its first call on a device looks up the buffer's
 *     device address with that device current; make that first call before
 *     any stream capture, and do not reset the device afterwards (the address
 *     is kept per device for the life of the process).
 *   - Every call shares the buffer and it keeps the last call's contents;
 *     nothing in it needs to start at zero (each call writes the scratch it
 *     reads).  Calls whose executions overlap on the GPU (other streams,
 *     other host threads) race on it and must be serialised by the caller.
 */
ssd_status ssd_scan_fwd_noalloc(const ssd_dims* d, const void* x, const float* dt, const float* A,
                                const void* Bm, const void* Cm, const float* D,
                                const float* init_state, void* y, float* final_state,
                                void* stream);

/*
 * Step 1, the log-decay cumulative sum ("分块推理…" §2.2, the product of A_t over a
 * chunk, taken in log space):  lam[b,h,c,i] = sum_{r=0..i} dt[b,cQ+r,h] * A[h]
 * for i < len(c); positions past the end of a short last chunk repeat the
 * chunk total.  Summed sequentially in fp32 so that differences
 * lam[t] - lam[s] keep their accuracy.
 */
ssd_status ssd_chunk_cumsum(const ssd_dims* d, const float* dt, const float* A, float* lam,
                            void* stream);

/*
 * Step 2, chunk-local states from a zero start ("分块推理…" §2.1, b_intra):
 *   chunk_states[b,h,c,n,p] = sum_{s in c} exp(lam_end(c) - lam_s) Bm[b,s,g,n] x[b,s,h,p]
 * (fp32 accumulation; tensor cores for bf16 io where supported).
 */
ssd_status ssd_chunk_state(const ssd_dims* d, const void* x, const void* Bm, const float* lam,
                           float* chunk_states, void* stream);

/*
 * Step 3, the inter-chunk recursion ("分块推理…" §2.2):
 *   b(-1) = init_state (or 0);  b(c) = chunk_states(c) + exp(lam_end(c)) b(c-1)
 * writes prev_states(c) = b(c-1) for every chunk and final_state = b(nc-1).
 * prev_states may alias chunk_states (updated in place); final_state may be
 * NULL and may alias init_state.
 */
ssd_status ssd_state_passing(const ssd_dims* d, const float* chunk_states, const float* lam,
                             const float* init_state, float* prev_states, float* final_state,
                             void* stream);

/*
 * Step 4, chunk outputs ("分块推理…" §2.1-§2.2, y = by_intra + by_inter):
 *   y_t = sum_{s<=t, s in c} (C_t . B_s) exp(lam_t - lam_s) x_s
 *       + exp(lam_t) C_t^T prev_states(c) + D[h] x_t
 */
ssd_status ssd_chunk_scan(const ssd_dims* d, const void* x, const void* Bm, const void* Cm,
                          const float* lam, const float* D, const float* prev_states, void* y,
                          void* stream);

/*
 * Layer-to-layer normalisation of the multi-layer stack (a reading: the
 * pages only say that layer l's output feeds layer l+1):
 *   out[r,:] = in[r,:] / sqrt(mean_f in[r,f]^2 + eps), computed in fp32,
 * for `rows` rows of `features` contiguous values; in/out in `io_dtype`
 * (may alias).
 */
ssd_status ssd_rmsnorm(int64_t rows, int64_t features, int32_t io_dtype, const void* in, float eps,
                       void* out, void* stream);

/*
 * One layer of a stack with the layer-to-layer RMS norm fused into the scan
 * (the normalisation of ssd_rmsnorm, but the normalised input is never
 * stored): the scan of x'_t = r_t x_t with
 *   r_t = 1 / sqrt(sum_h ss_in[b,t,h] / (H P) + rms_eps),
 * where x is the previous layer's stored y and ss_in[b,t,h] = sum_p x[b,t,h,p]^2
 * (as the previous call wrote to its ss_out).  The skip term is D_h x'_t.
 *   x, dt, A, Bm, Cm, D, init_state, y, final_state: as ssd_scan_fwd;
 *   ss_in [B,L,H] f32 or NULL (x is used as is: the stack's first layer);
 *   ss_out [B,L,H] f32 or NULL: ss_out[b,t,h] = sum_p y[b,t,h,p]^2 over the
 *   stored (io dtype) values of this call's y, for the next layer.
 * Takes the one-head tensor-core kernel only (bf16, P = 64, N = 128, Q a
 * multiple of 128; flags 0 or SSD_FLAG_INPUT_DT), else SSD_ERR_UNSUPPORTED.
 * ss_in, ss_out 16-byte aligned, not overlapping x, y or each other; no
 * workspace.  Layers chained through it give the results of ssd_vertical_fwd
 * with vblock >= L bitwise.
 */
ssd_status ssd_scan_fwd_normed(const ssd_dims* d, const void* x, const float* ss_in, float rms_eps,
                               const float* dt, const float* A, const void* Bm, const void* Cm,
                               const float* D, const float* init_state, void* y, float* ss_out,
                               float* final_state, void* stream);

/*
 * Bytes of workspace ssd_vertical_fwd needs for `d`, `n_layers` and the
 * vertical block length `vblock` (V): the single-block scan scratch plus two
 * V-token activation blocks per layer boundary ([B,V,H,P] io each; at least
 * two) and their per-(token, head) sums of squares ([B,V,H] f32 each).
 */
ssd_status ssd_vertical_workspace_size(const ssd_dims* d, int32_t n_layers, int64_t vblock,
                                       size_t* bytes);

/*
 * Depth-first multi-layer schedule, "分块推理…" §3.2: the sequence is cut into
 * V-token blocks; each block passes through layers 0..n_layers-1 before the
 * next block starts, and every layer keeps its state b between blocks.
 *   x0: layer-0 input [B,L,H,P] io.
 *   dt, A, Bm, Cm, D: HOST arrays of n_layers DEVICE pointers (D[l] may be
 *   NULL), each with the single-layer layout above.
 *   states: HOST array of n_layers DEVICE pointers [B,H,N,P] f32: the initial
 *   state of each layer on entry, its final state on return (in place).
 *   y_out: the last layer's output [B,L,H,P] io.
 * Layer l+1's input is y_l RMS-normalised over its H*P features (eps =
 * rms_eps).  With the one-head fused kernel the norm is fused: layer l writes
 * y_l and its per-(token, head) sums of squares, layer l+1 scales its input
 * rows on the fly (ssd_scan_fwd_normed), and no normalised copy is stored;
 * otherwise (SSD_FLAG_TWO_HEADS_PER_CTA, other shapes) layer l+1's input is
 * ssd_rmsnorm(y_l), stored in io dtype.
 * When V is a multiple of Q the result is bitwise equal to running the layers
 * one after another over the whole sequence (the §3.1 horizontal schedule):
 * ssd_scan_fwd_normed per layer, or ssd_scan_fwd and ssd_rmsnorm.
 * Execution: with more than one layer and a problem the fused tensor-core
 * kernel takes, the (block, layer) launches run as a wavefront: layer l on a
 * stream of its own, block k of layer l after block k of layer l-1, so
 * different layers' blocks overlap on the GPU.  Those streams and their
 * events belong to the library (one set per device, created on first use,
 * kept until the process exits); every call forks them from `stream` and
 * joins them back into it, so the call stays asynchronous, orders like a
 * single-stream call, and can be captured into a CUDA graph (make the first
 * call on a device outside a capture: it creates the streams and events).
 * Calls from several host threads on one device are serialised while they
 * enqueue.
 * Otherwise the blocks and layers run one after another on `stream`.
 */
ssd_status ssd_vertical_fwd(const ssd_dims* d, int32_t n_layers, int64_t vblock, float rms_eps,
                            const void* x0, const float* const* dt, const float* const* A,
                            const void* const* Bm, const void* const* Cm, const float* const* D,
                            float* const* states, void* y_out, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * Recurrent (decode) step: one token per (batch, head), the state updated in
 * place -- the token recurrence of "分块推理…" §2 itself, the mode a model runs
 * in when it generates with a state cache:
 *   a = exp(dt A_h);  state = a state + B x^T;  y = C^T state + D_h x
 *   d: sizes (seqlen and chunk are ignored), x [B,H,P] io, dt [B,H] f32,
 *   A [H] f32, Bm/Cm [B,G,N] io, D [H] f32 or NULL, state [B,H,N,P] f32
 *   (h_{t-1} on entry, h_t on return), y [B,H,P] io (must not overlap inputs).
 * Pointers need only their element's natural alignment (2 or 4 bytes), so a
 * token slice x[:, t] of a [B,L,H,P] tensor can be passed directly.
 * Errors: as ssd_scan_fwd except SSD_ERR_WORKSPACE (no workspace).
 */
ssd_status ssd_step(const ssd_dims* d, const void* x, const float* dt, const float* A, const void* Bm,
                    const void* Cm, const float* D, float* state, void* y, void* stream);

/*
 * The scan with a vector-valued decay: one decay rate per state channel n in
 * place of the per-head scalar -- the diagonal state matrix of the selective
 * scan ("告别Transformer的二次方噩梦…" §2.1) and the per-channel decays of the
 * recurrences "分块推理…" §6 names (RWKV, xLSTM):
 *     a_t[n] = exp(dt[b,t,h] * Av[h,n])
 *     h_t[n,:] = a_t[n] h_{t-1}[n,:] + Bm[b,t,g,n] x[b,t,h,:]
 *     y_t = Cm[b,t,g,:]^T h_t + D[h] x[b,t,h,:]
 *   Av: [H, N] f32 (non-positive); every other argument, layout and error as
 *   ssd_scan_fwd (fp32 or bf16 io), without a workspace; d->flags must be 0
 *   (else SSD_ERR_UNSUPPORTED).  Pointers need their element's natural
 *   alignment only.  Runs the token recurrence on CUDA cores (fp32 state):
 *   with channel-dependent decays the chunked form's intra-chunk term no
 *   longer factors into (C B^T) (.) L.  With Av[h,n] equal over n the result
 *   is ssd_scan_fwd's up to rounding.
 */
ssd_status ssd_scan_fwd_vdecay(const ssd_dims* d, const void* x, const float* dt, const float* Av, const void* Bm,
                               const void* Cm, const float* D, const float* init_state, void* y,
                               float* final_state, void* stream);

/*
 * Read and clear the device status word that bounded waits inside the
 * kernels set (synchronises `stream`).  Returns SSD_OK or SSD_ERR_TIMEOUT.
 */
ssd_status ssd_read_device_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SSD_B200_SSD_H */
