// Host side of libssd: argument validation, workspace carving and launch
// sequencing on the caller's stream for every entry point of include/ssd.h.
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "ssd_common.cuh"
#include "ssd_tc.cuh"

using namespace ssd;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned_to(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t io_size(int io) { return io == SSD_BF16 ? 2 : 4; }

ssd_status validate_dims(const ssd_dims* d) {
  if (!d) return SSD_ERR_INVALID_ARG;
  if ((d->flags & ~(SSD_FLAG_INPUT_DT | SSD_FLAG_TWO_HEADS_PER_CTA)) != 0) return SSD_ERR_INVALID_ARG;
  if (d->io_dtype != SSD_F32 && d->io_dtype != SSD_BF16) return SSD_ERR_DTYPE;
  if (d->batch < 1 || d->seqlen < 1 || d->nheads < 1 || d->headdim < 1 || d->dstate < 1 || d->ngroups < 1 ||
      d->chunk < 1)
    return SSD_ERR_SHAPE;
  if (d->nheads % d->ngroups != 0) return SSD_ERR_SHAPE;
  if (d->headdim > 64 || d->dstate > 128 || d->chunk > 256) return SSD_ERR_UNSUPPORTED;
  // grid limits: y = H, z = B (<= 65535); x = nc * ceil(Q/64) < 2^31
  const int64_t nc = ceil_div(d->seqlen, d->chunk);
  if (d->nheads > 65535 || d->batch > 65535 || nc * 4 >= (int64_t(1) << 31)) return SSD_ERR_UNSUPPORTED;
  return SSD_OK;
}

Problem make_problem(const ssd_dims* d) {
  Problem p;
  memset(&p, 0, sizeof(p));
  p.B = d->batch;
  p.L = d->seqlen;
  p.H = d->nheads;
  p.P = d->headdim;
  p.N = d->dstate;
  p.G = d->ngroups;
  p.Q = d->chunk;
  p.nc = ceil_div(p.L, p.Q);
  p.io = d->io_dtype;
  p.sx = p.L * p.H * p.P;
  p.sdt = p.L * p.H;
  p.sbc = p.L * p.G * p.N;
  p.sy = p.L * p.H * p.P;
  p.ldx = p.ldy = p.H * p.P;
  p.lddt = p.H;
  p.ldbc = p.G * p.N;
  p.input_dt = (d->flags & SSD_FLAG_INPUT_DT) ? 1 : 0;
  p.two_heads = (d->flags & SSD_FLAG_TWO_HEADS_PER_CTA) ? 1 : 0;
  return p;
}

struct Range {
  uintptr_t lo, hi;
};
Range range_of(const void* p, size_t bytes) {
  uintptr_t a = reinterpret_cast<uintptr_t>(p);
  return Range{a, a + bytes};
}
bool overlaps(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

// Workspace of the step-by-step path: lam [B,H,nc,Q] then states [B,H,nc,N,P].
size_t unfused_ws_bytes(const Problem& p) {
  return align_up(sizeof(float) * p.B * p.H * p.nc * p.Q) + align_up(sizeof(float) * p.B * p.H * p.nc * p.N * p.P);
}

ssd_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SSD_OK;
  fprintf(stderr, "libssd: CUDA error %d (%s)\n", (int)e, cudaGetErrorString(e));
  return SSD_ERR_CUDA;
}

ssd_status validate_scan_args(const ssd_dims* d, const void* x, const float* dt, const float* A, const void* Bm,
                              const void* Cm, const float* D, const float* init, const void* y,
                              const float* final_state, bool natural_alignment = false) {
  if (!x || !dt || !A || !Bm || !Cm || !y) return SSD_ERR_INVALID_ARG;
  const void* ptrs[] = {x, dt, A, Bm, Cm, D, init, y, final_state};
  const uintptr_t io_al = natural_alignment ? (d->io_dtype == SSD_BF16 ? 2 : 4) : 16;
  const uintptr_t f_al = natural_alignment ? 4 : 16;
  const bool is_io[] = {true, false, false, true, true, false, false, true, false};
  for (int i = 0; i < 9; ++i)
    if (ptrs[i] && !aligned_to(ptrs[i], is_io[i] ? io_al : f_al)) return SSD_ERR_ALIGN;
  const size_t es = io_size(d->io_dtype);
  const size_t nx = (size_t)d->batch * d->seqlen * d->nheads * d->headdim;
  const size_t nbc = (size_t)d->batch * d->seqlen * d->ngroups * d->dstate;
  const size_t nst = (size_t)d->batch * d->nheads * d->dstate * d->headdim;
  const Range ry = range_of(y, nx * es);
  const Range inputs[] = {range_of(x, nx * es),
                          range_of(dt, sizeof(float) * d->batch * d->seqlen * d->nheads),
                          range_of(A, sizeof(float) * d->nheads),
                          range_of(Bm, nbc * es),
                          range_of(Cm, nbc * es),
                          D ? range_of(D, sizeof(float) * d->nheads) : Range{0, 0},
                          init ? range_of(init, sizeof(float) * nst) : Range{0, 0},
                          final_state ? range_of(final_state, sizeof(float) * nst) : Range{0, 0}};
  for (const Range& r : inputs)
    if (r.hi > r.lo && overlaps(ry, r)) return SSD_ERR_INVALID_ARG;
  if (final_state && init && final_state != init &&
      overlaps(range_of(final_state, sizeof(float) * nst), range_of(init, sizeof(float) * nst)))
    return SSD_ERR_INVALID_ARG;
  return SSD_OK;
}

// The four step kernels in sequence over workspace (lam, states).
ssd_status run_unfused(const Problem& p, const float* init, float* final_state, char* ws, cudaStream_t st) {
  float* lam = reinterpret_cast<float*>(ws);
  float* states = reinterpret_cast<float*>(ws + align_up(sizeof(float) * p.B * p.H * p.nc * p.Q));
  cudaError_t e = launch_chunk_cumsum(p, lam, st);
  if (e == cudaSuccess) {
    if (tc_supported(p))
      e = launch_chunk_states_seq(p, lam, states, st);
    else
      e = launch_chunk_state_simt(p, lam, states, st);
  }
  if (e == cudaSuccess) e = launch_state_passing(p, states, lam, init, states, final_state, st);
  if (e == cudaSuccess) {
    if (tc_supported(p))
      e = launch_chunk_scan_tc(p, lam, states, st);
    else
      e = launch_chunk_scan_simt(p, lam, states, st);
  }
  return cuda_status(e);
}

}  // namespace

extern "C" {

const char* ssd_status_string(ssd_status s) {
  switch (s) {
    case SSD_OK: return "SSD_OK";
    case SSD_ERR_INVALID_ARG: return "SSD_ERR_INVALID_ARG: missing pointer, bad enum or overlapping buffers";
    case SSD_ERR_SHAPE: return "SSD_ERR_SHAPE: non-positive size or nheads not divisible by ngroups";
    case SSD_ERR_DTYPE: return "SSD_ERR_DTYPE: unsupported io dtype";
    case SSD_ERR_ALIGN: return "SSD_ERR_ALIGN: pointer not 16-byte aligned";
    case SSD_ERR_UNSUPPORTED: return "SSD_ERR_UNSUPPORTED: size outside the supported set";
    case SSD_ERR_WORKSPACE: return "SSD_ERR_WORKSPACE: workspace missing or too small";
    case SSD_ERR_CUDA: return "SSD_ERR_CUDA: a CUDA launch or query failed";
    case SSD_ERR_TIMEOUT: return "SSD_ERR_TIMEOUT: a bounded device-side wait gave up";
  }
  return "SSD_ERR_UNKNOWN";
}

int ssd_version(void) { return 100; }

ssd_status ssd_scan_workspace_size(const ssd_dims* d, size_t* bytes) {
  if (!bytes) return SSD_ERR_INVALID_ARG;
  ssd_status s = validate_dims(d);
  if (s != SSD_OK) return s;
  const Problem p = make_problem(d);
  size_t need = unfused_ws_bytes(p);
  const size_t tc = tc_workspace_bytes(p);
  if (tc > need) need = tc;
  *bytes = need;
  return SSD_OK;
}

ssd_status ssd_scan_path(const ssd_dims* d, int32_t* path, int32_t* kernels) {
  ssd_status s = validate_dims(d);
  if (s != SSD_OK) return s;
  const Problem p = make_problem(d);
  int32_t pa = SSD_PATH_CUDA_CORES, k = 4;
  if (fused_supported(p)) {
    pa = uses_pair_kernel(p) ? SSD_PATH_FUSED_PAIR : SSD_PATH_FUSED;
    k = fused_kernels_per_call(p);
  } else if (tc_supported(p)) {
    pa = SSD_PATH_TENSOR_STEPS;
  }
  if (path) *path = pa;
  if (kernels) *kernels = k;
  return SSD_OK;
}

ssd_status ssd_scan_fwd_unfused(const ssd_dims* d, const void* x, const float* dt, const float* A, const void* Bm,
                                const void* Cm, const float* D, const float* init_state, void* y,
                                float* final_state, void* workspace, size_t workspace_bytes, void* stream) {
  ssd_status s = validate_dims(d);
  if (s != SSD_OK) return s;
  s = validate_scan_args(d, x, dt, A, Bm, Cm, D, init_state, y, final_state);
  if (s != SSD_OK) return s;
  if (d->flags & SSD_FLAG_INPUT_DT) return SSD_ERR_UNSUPPORTED;  // the tensor-core path only
  Problem p = make_problem(d);
  if (!workspace || workspace_bytes < unfused_ws_bytes(p)) return SSD_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SSD_ERR_ALIGN;
  p.x = x; p.dt = dt; p.A = A; p.Bm = Bm; p.Cm = Cm; p.D = D; p.y = y;
  return run_unfused(p, init_state, final_state, static_cast<char*>(workspace), static_cast<cudaStream_t>(stream));
}

ssd_status ssd_scan_fwd(const ssd_dims* d, const void* x, const float* dt, const float* A, const void* Bm,
                        const void* Cm, const float* D, const float* init_state, void* y, float* final_state,
                        void* workspace, size_t workspace_bytes, void* stream) {
  ssd_status s = validate_dims(d);
  if (s != SSD_OK) return s;
  s = validate_scan_args(d, x, dt, A, Bm, Cm, D, init_state, y, final_state);
  if (s != SSD_OK) return s;
  Problem p = make_problem(d);
  size_t need = 0;
  ssd_scan_workspace_size(d, &need);
  if (!workspace || workspace_bytes < need) return SSD_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SSD_ERR_ALIGN;
  p.x = x; p.dt = dt; p.A = A; p.Bm = Bm; p.Cm = Cm; p.D = D; p.y = y;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (fused_supported(p))
    return cuda_status(launch_fused(p, init_state, final_state, workspace, workspace_bytes, st));
  if (p.input_dt) return SSD_ERR_UNSUPPORTED;  // the dt-scaled input: tensor-core path only
  return run_unfused(p, init_state, final_state, static_cast<char*>(workspace), st);
}

ssd_status ssd_scan_fwd_normed(const ssd_dims* d, const void* x, const float* ss_in, float rms_eps,
                               const float* dt, const float* A, const void* Bm, const void* Cm,
                               const float* D, const float* init_state, void* y, float* ss_out,
                               float* final_state, void* stream) {
  ssd_status s = validate_dims(d);
  if (s != SSD_OK) return s;
  if (d->flags & ~SSD_FLAG_INPUT_DT) return SSD_ERR_UNSUPPORTED;  // the one-head kernel only
  s = validate_scan_args(d, x, dt, A, Bm, Cm, D, init_state, y, final_state);
  if (s != SSD_OK) return s;
  Problem p = make_problem(d);
  if (!fused_supported(p)) return SSD_ERR_UNSUPPORTED;
  if (!(rms_eps >= 0.0f)) return SSD_ERR_INVALID_ARG;
  if ((ss_in && !aligned16(ss_in)) || (ss_out && !aligned16(ss_out))) return SSD_ERR_ALIGN;
  const size_t es = io_size(d->io_dtype);
  const size_t act = es * (size_t)p.B * p.L * p.H * p.P, sums = sizeof(float) * (size_t)p.B * p.L * p.H;
  const Range rx = range_of(x, act), ry = range_of(y, act);
  if (ss_in && (overlaps(range_of(ss_in, sums), rx) || overlaps(range_of(ss_in, sums), ry)))
    return SSD_ERR_INVALID_ARG;
  if (ss_out && (overlaps(range_of(ss_out, sums), rx) || overlaps(range_of(ss_out, sums), ry) ||
                 (ss_in && overlaps(range_of(ss_out, sums), range_of(ss_in, sums)))))
    return SSD_ERR_INVALID_ARG;
  p.x = x; p.dt = dt; p.A = A; p.Bm = Bm; p.Cm = Cm; p.D = D; p.y = y;
  NormIO nio;
  nio.ss_in = ss_in;
  nio.ss_out = ss_out;
  nio.batch_stride = p.L * p.H;
  nio.eps = rms_eps;
  return cuda_status(launch_fused_normed(p, init_state, final_state, nio, static_cast<cudaStream_t>(stream)));
}

ssd_status ssd_scan_fwd_strided(const ssd_dims* d, const void* x, int64_t x_bstride, int64_t x_tstride,
                                const float* dt, int64_t dt_bstride, int64_t dt_tstride, const float* A, const void* Bm,
                                const void* Cm, int64_t bc_bstride, int64_t bc_tstride, const float* D,
                                const float* init_state, void* y, int64_t y_bstride, int64_t y_tstride,
                                float* final_state, void* stream) {
  ssd_status s = validate_dims(d);
  if (s != SSD_OK) return s;
  Problem p = make_problem(d);
  if (!fused_supported(p)) return SSD_ERR_UNSUPPORTED;  // the tensor-core path only
  if (!x || !dt || !A || !Bm || !Cm || !y) return SSD_ERR_INVALID_ARG;
  const int64_t HP = p.H * p.P, GN = p.G * p.N;
  // a token's heads (groups) stay dense; tokens may be further apart, batches too
  if (x_tstride < HP || y_tstride < HP || dt_tstride < p.H || bc_tstride < GN) return SSD_ERR_SHAPE;
  if (x_bstride < (p.L - 1) * x_tstride + HP || y_bstride < (p.L - 1) * y_tstride + HP ||
      dt_bstride < (p.L - 1) * dt_tstride + p.H || bc_bstride < (p.L - 1) * bc_tstride + GN)
    return SSD_ERR_SHAPE;
  // TMA strides are multiples of 16 bytes: 8 bf16 elements
  if ((x_tstride | x_bstride | y_tstride | y_bstride | bc_tstride | bc_bstride) & 7) return SSD_ERR_ALIGN;
  if (!aligned16(x) || !aligned16(y) || !aligned16(Bm) || !aligned16(Cm) || !aligned16(A) ||
      (D && !aligned16(D)) || !aligned_to(dt, 4) || (init_state && !aligned16(init_state)) ||
      (final_state && !aligned16(final_state)))
    return SSD_ERR_ALIGN;
  // y must not overlap an input (extents from first to last element touched)
  const size_t es = io_size(d->io_dtype);
  const Range ry = range_of(y, es * (size_t)((p.B - 1) * y_bstride + (p.L - 1) * y_tstride + HP));
  const Range rin[] = {range_of(x, es * (size_t)((p.B - 1) * x_bstride + (p.L - 1) * x_tstride + HP)),
                       range_of(Bm, es * (size_t)((p.B - 1) * bc_bstride + (p.L - 1) * bc_tstride + GN)),
                       range_of(Cm, es * (size_t)((p.B - 1) * bc_bstride + (p.L - 1) * bc_tstride + GN)),
                       range_of(dt, 4 * (size_t)((p.B - 1) * dt_bstride + (p.L - 1) * dt_tstride + p.H))};
  for (const Range& r : rin)
    if (overlaps(ry, r)) return SSD_ERR_INVALID_ARG;
  p.x = x; p.dt = dt; p.A = A; p.Bm = Bm; p.Cm = Cm; p.D = D; p.y = y;
  p.sx = x_bstride; p.ldx = x_tstride;
  p.sdt = dt_bstride; p.lddt = dt_tstride;
  p.sbc = bc_bstride; p.ldbc = bc_tstride;
  p.sy = y_bstride; p.ldy = y_tstride;
  return cuda_status(launch_fused(p, init_state, final_state, nullptr, 0, static_cast<cudaStream_t>(stream)));
}

ssd_status ssd_chunk_cumsum(const ssd_dims* d, const float* dt, const float* A, float* lam, void* stream) {
  ssd_status s = validate_dims(d);
  if (s != SSD_OK) return s;
  if (d->flags & SSD_FLAG_INPUT_DT) return SSD_ERR_UNSUPPORTED;
  if (!dt || !A || !lam) return SSD_ERR_INVALID_ARG;
  if (!aligned16(dt) || !aligned16(A) || !aligned16(lam)) return SSD_ERR_ALIGN;
  Problem p = make_problem(d);
  p.dt = dt; p.A = A;
  return cuda_status(launch_chunk_cumsum(p, lam, static_cast<cudaStream_t>(stream)));
}

ssd_status ssd_chunk_state(const ssd_dims* d, const void* x, const void* Bm, const float* lam, float* chunk_states,
                           void* stream) {
  ssd_status s = validate_dims(d);
  if (s != SSD_OK) return s;
  if (d->flags & SSD_FLAG_INPUT_DT) return SSD_ERR_UNSUPPORTED;
  if (!x || !Bm || !lam || !chunk_states) return SSD_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(Bm) || !aligned16(lam) || !aligned16(chunk_states)) return SSD_ERR_ALIGN;
  Problem p = make_problem(d);
  p.x = x; p.Bm = Bm;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc_supported(p)) return cuda_status(launch_chunk_states_seq(p, lam, chunk_states, st));
  return cuda_status(launch_chunk_state_simt(p, lam, chunk_states, st));
}

ssd_status ssd_state_passing(const ssd_dims* d, const float* chunk_states, const float* lam, const float* init_state,
                             float* prev_states, float* final_state, void* stream) {
  ssd_status s = validate_dims(d);
  if (s != SSD_OK) return s;
  if (d->flags & SSD_FLAG_INPUT_DT) return SSD_ERR_UNSUPPORTED;
  if (!chunk_states || !lam || !prev_states) return SSD_ERR_INVALID_ARG;
  const void* ptrs[] = {chunk_states, lam, init_state, prev_states, final_state};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return SSD_ERR_ALIGN;
  Problem p = make_problem(d);
  return cuda_status(launch_state_passing(p, chunk_states, lam, init_state, prev_states, final_state,
                                          static_cast<cudaStream_t>(stream)));
}

ssd_status ssd_chunk_scan(const ssd_dims* d, const void* x, const void* Bm, const void* Cm, const float* lam,
                          const float* D, const float* prev_states, void* y, void* stream) {
  ssd_status s = validate_dims(d);
  if (s != SSD_OK) return s;
  if (d->flags & SSD_FLAG_INPUT_DT) return SSD_ERR_UNSUPPORTED;
  if (!x || !Bm || !Cm || !lam || !prev_states || !y) return SSD_ERR_INVALID_ARG;
  const void* ptrs[] = {x, Bm, Cm, lam, D, prev_states, y};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return SSD_ERR_ALIGN;
  Problem p = make_problem(d);
  p.x = x; p.Bm = Bm; p.Cm = Cm; p.D = D; p.y = y;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (tc_supported(p)) return cuda_status(launch_chunk_scan_tc(p, lam, prev_states, st));
  return cuda_status(launch_chunk_scan_simt(p, lam, prev_states, st));
}

ssd_status ssd_rmsnorm(int64_t rows, int64_t features, int32_t io_dtype, const void* in, float eps, void* out,
                       void* stream) {
  if (rows < 0 || features < 1) return SSD_ERR_SHAPE;
  if (io_dtype != SSD_F32 && io_dtype != SSD_BF16) return SSD_ERR_DTYPE;
  if (rows > 0x7fffffff) return SSD_ERR_UNSUPPORTED;
  if (rows > 0 && (!in || !out)) return SSD_ERR_INVALID_ARG;
  if ((in && !aligned16(in)) || (out && !aligned16(out))) return SSD_ERR_ALIGN;
  if (!(eps >= 0.0f)) return SSD_ERR_INVALID_ARG;
  return cuda_status(launch_rmsnorm(rows, features, io_dtype, in, eps, out, static_cast<cudaStream_t>(stream)));
}

// Vertical (depth-first) schedule.  Workspace: the single-layer workspace of
// a V-token slice, then the activation blocks [B, V, H, P] (io dtype) and, for
// the fused RMS norm, their per-(token, head) sums of squares [B, V, H] f32.
ssd_status ssd_vertical_workspace_size(const ssd_dims* d, int32_t n_layers, int64_t vblock, size_t* bytes) {
  if (!bytes) return SSD_ERR_INVALID_ARG;
  ssd_status s = validate_dims(d);
  if (s != SSD_OK) return s;
  if (n_layers < 1 || vblock < 1) return SSD_ERR_SHAPE;
  ssd_dims dv = *d;
  dv.seqlen = vblock < d->seqlen ? vblock : d->seqlen;
  size_t one = 0;
  s = ssd_scan_workspace_size(&dv, &one);
  if (s != SSD_OK) return s;
  const size_t act = align_up(io_size(d->io_dtype) * (size_t)d->batch * dv.seqlen * d->nheads * d->headdim);
  // the wavefront schedule keeps two activation blocks per layer boundary
  const size_t nact = n_layers > 2 ? 2 * (size_t)(n_layers - 1) : 2;
  const size_t sums = align_up(sizeof(float) * (size_t)d->batch * dv.seqlen * d->nheads);
  *bytes = align_up(one) + nact * (act + sums);
  return SSD_OK;
}

namespace {

// Streams and events of the wavefront schedule, one set per device, created on
// first use and kept for the life of the process.  `mu` is held while a call
// enqueues its work, so calls from several host threads never interleave
// their event records.
struct WavefrontPool {
  std::mutex mu;
  std::vector<cudaStream_t> streams;  // one per layer
  std::vector<cudaEvent_t> out;       // [layer]: block's output of that layer is normalised and ready
  std::vector<cudaEvent_t> freed;     // [layer][2]: the layer finished reading its input buffer of that parity
  cudaEvent_t fork = nullptr;

  cudaError_t grow(int n) {
    if (!fork) {
      cudaError_t e = cudaEventCreateWithFlags(&fork, cudaEventDisableTiming);
      if (e != cudaSuccess) return e;
    }
    while ((int)streams.size() < n) {
      cudaStream_t s;
      cudaEvent_t a, b, c;
      cudaError_t e = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&a, cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&b, cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c, cudaEventDisableTiming);
      if (e != cudaSuccess) return e;
      streams.push_back(s);
      out.push_back(a);
      freed.push_back(b);
      freed.push_back(c);
    }
    return cudaSuccess;
  }
};

WavefrontPool* wavefront_pool(int device) {
  static std::mutex mu;
  static std::vector<WavefrontPool*> pools;
  std::lock_guard<std::mutex> lock(mu);
  if (device < 0) return nullptr;
  if ((int)pools.size() <= device) pools.resize(device + 1, nullptr);
  if (!pools[device]) pools[device] = new WavefrontPool();
  return pools[device];
}

}  // namespace

// Wavefront form of the depth-first schedule (fused kernel only: it needs no
// scratch, so launches of different layers may run at the same time).  Layer
// l runs on its own stream, blocks in order, so its state passes from block k
// to block k+1 by stream order.  Block k of layer l waits for block k of layer
// l-1 (its input, normalised) and, before it overwrites the input buffer of
// layer l+1 of parity k % 2, for layer l+1 to have finished block k-2 (the
// last reader of that buffer).  Every (block, layer) runs the same kernel on
// the same data as the one-block-at-a-time order, so results are identical.
static ssd_status vertical_wavefront(const ssd_dims* d_, int32_t n_layers, int64_t V, float rms_eps, const void* x0,
                                     const float* const* dt, const float* const* A, const void* const* Bm,
                                     const void* const* Cm, const float* const* D, float* const* states, void* y_out,
                                     void* workspace, cudaStream_t st) {
  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return cuda_status(e);
  WavefrontPool* pool = wavefront_pool(device);
  std::lock_guard<std::mutex> lock(pool->mu);
  e = pool->grow(n_layers);
  if (e != cudaSuccess) return cuda_status(e);

  const Problem full = make_problem(d_);
  ssd_dims dv = *d_;
  dv.seqlen = V;
  size_t one = 0;
  ssd_scan_workspace_size(&dv, &one);
  const size_t es = io_size(d_->io_dtype);
  const size_t act = align_up(es * (size_t)d_->batch * V * d_->nheads * d_->headdim);
  const size_t sums = align_up(sizeof(float) * (size_t)d_->batch * V * d_->nheads);
  char* ring = static_cast<char*>(workspace) + align_up(one);
  // input buffer of layer l (1 <= l < n_layers) for blocks of parity q, and its
  // rows' per-(token, head) sums of squares
  auto in_buf = [&](int l, int64_t q) { return ring + ((size_t)(l - 1) * 2 + (size_t)q) * (act + sums); };
  auto in_sums = [&](int l, int64_t q) { return reinterpret_cast<float*>(in_buf(l, q) + act); };
  const int64_t HP = full.H * full.P;

  // fork: every layer stream starts after the work already on `st`
  e = cudaEventRecord(pool->fork, st);
  for (int l = 0; l < n_layers && e == cudaSuccess; ++l) e = cudaStreamWaitEvent(pool->streams[l], pool->fork, 0);
  if (e != cudaSuccess) return cuda_status(e);

  // Enqueued by anti-diagonals d = k + l (the order the wavefront runs in), so
  // that the hardware queues the layer streams share never hold a wait in
  // front of work that is already runnable; inside a diagonal the layers go
  // downwards, so each wait binds to the record it means: block k of layer l
  // waits for block k of layer l-1, which block k+1 of layer l-1 (same
  // diagonal) re-records only afterwards.
  ssd_status s = SSD_OK;
  const int64_t nblk = (full.L + V - 1) / V;
  for (int64_t d = 0; d < nblk + n_layers - 1 && s == SSD_OK; ++d) {
    const int l_hi = (int)(d < n_layers - 1 ? d : n_layers - 1);
    const int l_lo = (int)(d - (nblk - 1) > 0 ? d - (nblk - 1) : 0);
    for (int l = l_hi; l >= l_lo; --l) {
      const int64_t k = d - l;
      const int64_t k0 = k * V;
      const int64_t Vk = (full.L - k0) < V ? (full.L - k0) : V;
      ssd_dims dk = *d_;
      dk.seqlen = Vk;
      cudaStream_t sl = pool->streams[l];
      const bool last = (l == n_layers - 1);
      Problem p = make_problem(&dk);
      if (l == 0) {
        p.x = static_cast<const char*>(x0) + es * k0 * HP;
        p.sx = full.L * HP;
      } else {
        p.x = in_buf(l, k & 1);
        p.sx = Vk * HP;
        e = cudaStreamWaitEvent(sl, pool->out[l - 1], 0);  // input of this block is ready
      }
      if (e == cudaSuccess && !last && k >= 2)  // layer l+1 is done with block k-2's buffer
        e = cudaStreamWaitEvent(sl, pool->freed[2 * (l + 1) + (k & 1)], 0);
      if (e != cudaSuccess) {
        s = cuda_status(e);
        break;
      }
      p.dt = dt[l] + k0 * full.H;
      p.sdt = full.L * full.H;
      p.A = A[l];
      p.Bm = static_cast<const char*>(Bm[l]) + es * k0 * full.G * full.N;
      p.Cm = static_cast<const char*>(Cm[l]) + es * k0 * full.G * full.N;
      p.sbc = full.L * full.G * full.N;
      p.D = D ? D[l] : nullptr;
      if (last) {
        p.y = static_cast<char*>(y_out) + es * k0 * HP;
        p.sy = full.L * HP;
      } else {
        p.y = in_buf(l + 1, k & 1);
        p.sy = Vk * HP;
      }
      if (uses_pair_kernel(p)) {  // the two-head kernel: the norm as its own pass
        s = cuda_status(launch_fused(p, states[l], states[l], nullptr, 0, sl));
        if (s == SSD_OK && !last)
          s = cuda_status(launch_rmsnorm(d_->batch * Vk, HP, d_->io_dtype, p.y, rms_eps, p.y, sl));
      } else {  // the norm fused: sums out of layer l, scales into layer l+1
        NormIO nio;
        nio.ss_in = l > 0 ? in_sums(l, k & 1) : nullptr;
        nio.ss_out = last ? nullptr : in_sums(l + 1, k & 1);
        nio.batch_stride = Vk * full.H;
        nio.eps = rms_eps;
        s = cuda_status(launch_fused_normed(p, states[l], states[l], nio, sl));
      }
      if (s != SSD_OK) break;
      e = cudaEventRecord(pool->out[l], sl);
      if (e == cudaSuccess && l > 0) e = cudaEventRecord(pool->freed[2 * l + (k & 1)], sl);
      if (e != cudaSuccess) {
        s = cuda_status(e);
        break;
      }
    }
  }
  // join: `st` continues after every layer stream (also after a failed launch,
  // so that no stream is left forked from a capture)
  for (int l = 0; l < n_layers; ++l) {
    cudaError_t ej = cudaEventRecord(pool->out[l], pool->streams[l]);
    if (ej == cudaSuccess) ej = cudaStreamWaitEvent(st, pool->out[l], 0);
    if (ej != cudaSuccess && s == SSD_OK) s = cuda_status(ej);
  }
  return s;
}

ssd_status ssd_vertical_fwd(const ssd_dims* d, int32_t n_layers, int64_t vblock, float rms_eps, const void* x0,
                            const float* const* dt, const float* const* A, const void* const* Bm,
                            const void* const* Cm, const float* const* D, float* const* states, void* y_out,
                            void* workspace, size_t workspace_bytes, void* stream) {
  ssd_status s = validate_dims(d);
  if (s != SSD_OK) return s;
  if (n_layers < 1 || vblock < 1) return SSD_ERR_SHAPE;
  if (!x0 || !dt || !A || !Bm || !Cm || !states || !y_out) return SSD_ERR_INVALID_ARG;
  if (!(rms_eps >= 0.0f)) return SSD_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l) {
    s = validate_scan_args(d, x0, dt[l], A[l], Bm[l], Cm[l], D ? D[l] : nullptr, states[l], y_out, states[l]);
    if (s != SSD_OK) return s;
    if (!states[l]) return SSD_ERR_INVALID_ARG;
  }
  size_t need = 0;
  s = ssd_vertical_workspace_size(d, n_layers, vblock, &need);
  if (s != SSD_OK) return s;
  if (!workspace || workspace_bytes < need) return SSD_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SSD_ERR_ALIGN;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Problem full = make_problem(d);
  if (full.input_dt && !fused_supported(full)) return SSD_ERR_UNSUPPORTED;
  const int64_t V = vblock < d->seqlen ? vblock : d->seqlen;
  if (n_layers > 1 && fused_supported(full))
    return vertical_wavefront(d, n_layers, V, rms_eps, x0, dt, A, Bm, Cm, D, states, y_out, workspace, st);
  ssd_dims dv = *d;
  dv.seqlen = V;
  size_t one = 0;
  ssd_scan_workspace_size(&dv, &one);
  char* ws = static_cast<char*>(workspace);
  const size_t es = io_size(d->io_dtype);
  const size_t act = align_up(es * (size_t)d->batch * V * d->nheads * d->headdim);
  char* buf[2] = {ws + align_up(one), ws + align_up(one) + act};
  const int64_t HP = full.H * full.P;

  for (int64_t k0 = 0; k0 < full.L; k0 += V) {
    const int64_t Vk = (full.L - k0) < V ? (full.L - k0) : V;
    ssd_dims dk = *d;
    dk.seqlen = Vk;
    Problem p = make_problem(&dk);
    for (int l = 0; l < n_layers; ++l) {
      // layer input: x0 slice for layer 0, else the normalised previous output
      if (l == 0) {
        p.x = static_cast<const char*>(x0) + es * k0 * HP;
        p.sx = full.L * HP;
      } else {
        p.x = buf[l & 1];
        p.sx = Vk * HP;
      }
      p.dt = dt[l] + k0 * full.H;
      p.sdt = full.L * full.H;
      p.A = A[l];
      p.Bm = static_cast<const char*>(Bm[l]) + es * k0 * full.G * full.N;
      p.Cm = static_cast<const char*>(Cm[l]) + es * k0 * full.G * full.N;
      p.sbc = full.L * full.G * full.N;
      p.D = D ? D[l] : nullptr;
      const bool last = (l == n_layers - 1);
      if (last) {
        p.y = static_cast<char*>(y_out) + es * k0 * HP;
        p.sy = full.L * HP;
      } else {
        p.y = buf[(l + 1) & 1];
        p.sy = Vk * HP;
      }
      if (fused_supported(p))
        s = cuda_status(launch_fused(p, states[l], states[l], nullptr, 0, st));
      else
        s = run_unfused(p, states[l], states[l], ws, st);
      if (s != SSD_OK) return s;
      if (!last) {
        s = cuda_status(launch_rmsnorm(d->batch * Vk, HP, d->io_dtype, p.y, rms_eps, p.y, st));
        if (s != SSD_OK) return s;
      }
    }
  }
  return SSD_OK;
}

ssd_status ssd_step(const ssd_dims* d, const void* x, const float* dt, const float* A, const void* Bm, const void* Cm,
                    const float* D, float* state, void* y, void* stream) {
  if (!d) return SSD_ERR_INVALID_ARG;
  ssd_dims d1 = *d;
  d1.seqlen = 1;
  d1.chunk = 1;
  ssd_status s = validate_dims(&d1);
  if (s != SSD_OK) return s;
  if (!state) return SSD_ERR_INVALID_ARG;
  s = validate_scan_args(&d1, x, dt, A, Bm, Cm, D, state, y, state, /*natural_alignment=*/true);
  if (s != SSD_OK) return s;
  Problem p = make_problem(&d1);
  p.x = x; p.dt = dt; p.A = A; p.Bm = Bm; p.Cm = Cm; p.D = D; p.y = y;
  return cuda_status(launch_ssd_step(p, state, static_cast<cudaStream_t>(stream)));
}

ssd_status ssd_read_device_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int h = 0;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&h, g_device_status, sizeof(int));
  if (e != cudaSuccess) return cuda_status(e);
  if (h != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_status(e);
    return SSD_ERR_TIMEOUT;
  }
  return SSD_OK;
}

}  // extern "C"
