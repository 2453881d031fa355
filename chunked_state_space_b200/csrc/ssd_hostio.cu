// ssd_scan_fwd_host: the scan from and to host memory, with the copies
// overlapped with the scan.
//
// The batch is cut into slices of one sequence and up to kSliceTokens tokens
// that flow through two device buffers: while slice s is scanned on the
// caller's stream, slice s+1 is copied in on a host-to-device stream and
// slice s-1 copied out on a device-to-host stream (the two directions use
// separate copy engines).  A buffer is refilled only after the copy-out of
// the slice it held.  The slices of one sequence are scanned in order, each
// from the end state of the one before (the page's chunk recursion with the
// slice as the chunk), so short slices keep the copy engines busy from the
// first slice to the last without changing the result beyond rounding: each
// slice runs the same launch as ssd_scan_fwd on its one-sequence problem.
// The copy streams and events belong to the library (one set per device,
// created on first use, kept until the process exits); every call forks them
// from the caller's stream and joins them back.
#include <mutex>
#include <vector>

#include "ssd_common.cuh"

namespace ssd {
namespace hostio {

struct Pool {
  std::mutex mu;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  cudaEvent_t in_ready[2] = {nullptr, nullptr};   // slice copied in
  cudaEvent_t scanned[2] = {nullptr, nullptr};    // slice scanned
  cudaEvent_t out_done[2] = {nullptr, nullptr};   // slice copied out: buffer free

  cudaError_t init() {
    if (h2d) return cudaSuccess;
    cudaError_t e = cudaStreamCreateWithFlags(&h2d, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&d2h, cudaStreamNonBlocking);
    cudaEvent_t* evs[] = {&fork, &join, &in_ready[0], &in_ready[1], &scanned[0], &scanned[1], &out_done[0],
                          &out_done[1]};
    for (cudaEvent_t* ev : evs)
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    if (e != cudaSuccess) h2d = nullptr;  // retried on the next call
    return e;
  }
};

static Pool* pool(int device) {
  static std::mutex mu;
  static std::vector<Pool*> pools;
  std::lock_guard<std::mutex> lock(mu);
  if (device < 0) return nullptr;
  if ((int)pools.size() <= device) pools.resize(device + 1, nullptr);
  if (!pools[device]) pools[device] = new Pool();
  return pools[device];
}

// Tokens per slice: long sequences are cut into slices of this length (a
// multiple of every supported chunk length up to it; shorter sequences are one
// slice), so the first copy-in and the last copy-out, which overlap nothing,
// are short.
constexpr int64_t kSliceTokens = 4096;

// Device workspace: A and D, then two slice buffers (x, dt, B, C, init, y,
// final, and the one-slice scan's scratch), each piece 256-byte aligned.
struct Layout {
  int64_t slice;                   // tokens per slice
  size_t x, dt, bc, st, scratch;   // bytes of one slice's pieces
  size_t off_a, off_d, slice0, slice_bytes, total;
  size_t o_x, o_dt, o_b, o_c, o_init, o_y, o_fin, o_scr;  // offsets inside a slice buffer
};

static int64_t slice_tokens(const ssd_dims* d) {
  if (d->seqlen <= kSliceTokens) return d->seqlen;
  const int64_t q = d->chunk > 0 ? d->chunk : 1;  // whole chunks per slice
  const int64_t t = kSliceTokens / q * q;
  return t > 0 ? t : q;
}

static ssd_status layout(const ssd_dims* d, Layout* lo) {
  ssd_dims d1 = *d;
  d1.batch = 1;
  d1.seqlen = slice_tokens(d);
  size_t one = 0;
  ssd_status s = ssd_scan_workspace_size(&d1, &one);
  if (s != SSD_OK) return s;
  const size_t es = io_size(d->io_dtype);
  lo->slice = d1.seqlen;
  lo->x = es * (size_t)d1.seqlen * d->nheads * d->headdim;
  lo->dt = sizeof(float) * (size_t)d1.seqlen * d->nheads;
  lo->bc = es * (size_t)d1.seqlen * d->ngroups * d->dstate;
  lo->st = sizeof(float) * (size_t)d->nheads * d->dstate * d->headdim;
  lo->scratch = one;
  size_t o = 0;
  lo->o_x = o;    o += align_up(lo->x);
  lo->o_dt = o;   o += align_up(lo->dt);
  lo->o_b = o;    o += align_up(lo->bc);
  lo->o_c = o;    o += align_up(lo->bc);
  lo->o_init = o; o += align_up(lo->st);
  lo->o_y = o;    o += align_up(lo->x);
  lo->o_fin = o;  o += align_up(lo->st);
  lo->o_scr = o;  o += align_up(lo->scratch > 0 ? lo->scratch : 1);
  lo->slice_bytes = o;
  lo->off_a = 0;
  lo->off_d = align_up(sizeof(float) * (size_t)d->nheads);
  lo->slice0 = lo->off_d + align_up(sizeof(float) * (size_t)d->nheads);
  lo->total = lo->slice0 + 2 * lo->slice_bytes;
  return SSD_OK;
}

}  // namespace hostio
}  // namespace ssd

extern "C" {

ssd_status ssd_scan_fwd_host_workspace_size(const ssd_dims* d, size_t* bytes) {
  using namespace ssd;
  if (!bytes) return SSD_ERR_INVALID_ARG;
  ssd_status s = validate_dims(d);
  if (s != SSD_OK) return s;
  hostio::Layout lo;
  s = hostio::layout(d, &lo);
  if (s != SSD_OK) return s;
  *bytes = lo.total;
  return SSD_OK;
}

ssd_status ssd_scan_fwd_host(const ssd_dims* d, const void* x, const float* dt, const float* A, const void* Bm,
                             const void* Cm, const float* D, const float* init_state, void* y, float* final_state,
                             void* workspace, size_t workspace_bytes, void* stream) {
  using namespace ssd;
  ssd_status s = validate_dims(d);
  if (s != SSD_OK) return s;
  if (!x || !dt || !A || !Bm || !Cm || !y) return SSD_ERR_INVALID_ARG;
  hostio::Layout lo;
  s = hostio::layout(d, &lo);
  if (s != SSD_OK) return s;
  if (!workspace || workspace_bytes < lo.total) return SSD_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SSD_ERR_ALIGN;

  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return cuda_status(e);
  hostio::Pool* pl = hostio::pool(device);
  std::lock_guard<std::mutex> lock(pl->mu);
  e = pl->init();
  if (e != cudaSuccess) return cuda_status(e);

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  float* dA = reinterpret_cast<float*>(ws + lo.off_a);
  float* dD = D ? reinterpret_cast<float*>(ws + lo.off_d) : nullptr;
  const char* hx = static_cast<const char*>(x);
  const char* hB = static_cast<const char*>(Bm);
  const char* hC = static_cast<const char*>(Cm);
  char* hy = static_cast<char*>(y);

  // fork the copy streams from the caller's stream
  e = cudaEventRecord(pl->fork, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(pl->h2d, pl->fork, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(pl->d2h, pl->fork, 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dA, A, sizeof(float) * d->nheads, cudaMemcpyHostToDevice, pl->h2d);
  if (e == cudaSuccess && D) e = cudaMemcpyAsync(dD, D, sizeof(float) * d->nheads, cudaMemcpyHostToDevice, pl->h2d);
  if (e != cudaSuccess) return cuda_status(e);

  // element strides of one token of one sequence
  const int64_t HP = d->nheads * d->headdim, GN = d->ngroups * d->dstate;
  const size_t es = io_size(d->io_dtype);
  const int64_t nsl = (d->seqlen + lo.slice - 1) / lo.slice;  // slices per sequence
  const size_t nst = lo.st / sizeof(float);
  for (int64_t sidx = 0; sidx < d->batch * nsl && s == SSD_OK; ++sidx) {
    const int64_t b = sidx / nsl, k = sidx % nsl;
    const int64_t t0 = k * lo.slice, len = (d->seqlen - t0) < lo.slice ? (d->seqlen - t0) : lo.slice;
    const int64_t tok = b * d->seqlen + t0;  // first token row of the slice in the batch
    const int kb = (int)(sidx & 1);
    char* buf = ws + lo.slice0 + (size_t)kb * lo.slice_bytes;
    char* prev = ws + lo.slice0 + (size_t)(kb ^ 1) * lo.slice_bytes;  // buffer of slice sidx-1
    const bool first = (k == 0), last = (k == nsl - 1);
    // copy in (after the copy-out of the slice that held this buffer)
    if (sidx >= 2) e = cudaStreamWaitEvent(pl->h2d, pl->out_done[kb], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(buf + lo.o_x, hx + tok * HP * es, (size_t)len * HP * es, cudaMemcpyHostToDevice, pl->h2d);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(buf + lo.o_dt, dt + tok * d->nheads, sizeof(float) * (size_t)len * d->nheads,
                          cudaMemcpyHostToDevice, pl->h2d);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(buf + lo.o_b, hB + tok * GN * es, (size_t)len * GN * es, cudaMemcpyHostToDevice, pl->h2d);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(buf + lo.o_c, hC + tok * GN * es, (size_t)len * GN * es, cudaMemcpyHostToDevice, pl->h2d);
    if (e == cudaSuccess && first && init_state)
      e = cudaMemcpyAsync(buf + lo.o_init, init_state + b * nst, lo.st, cudaMemcpyHostToDevice, pl->h2d);
    if (e == cudaSuccess) e = cudaEventRecord(pl->in_ready[kb], pl->h2d);
    // scan on the caller's stream, from the caller's initial state or the end
    // state of the slice before
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, pl->in_ready[kb], 0);
    if (e != cudaSuccess) {
      s = cuda_status(e);
      break;
    }
    ssd_dims d1 = *d;
    d1.batch = 1;
    d1.seqlen = len;
    const float* sinit = first ? (init_state ? reinterpret_cast<const float*>(buf + lo.o_init) : nullptr)
                               : reinterpret_cast<const float*>(prev + lo.o_fin);
    float* dfin = reinterpret_cast<float*>(buf + lo.o_fin);
    const bool need_fin = !last || final_state;
    s = ssd_scan_fwd(&d1, buf + lo.o_x, reinterpret_cast<const float*>(buf + lo.o_dt), dA, buf + lo.o_b,
                     buf + lo.o_c, dD, sinit, buf + lo.o_y, need_fin ? dfin : nullptr, buf + lo.o_scr,
                     lo.slice_bytes - lo.o_scr, st);
    if (s != SSD_OK) break;
    e = cudaEventRecord(pl->scanned[kb], st);
    // copy out
    if (e == cudaSuccess) e = cudaStreamWaitEvent(pl->d2h, pl->scanned[kb], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(hy + tok * HP * es, buf + lo.o_y, (size_t)len * HP * es, cudaMemcpyDeviceToHost, pl->d2h);
    if (e == cudaSuccess && last && final_state)
      e = cudaMemcpyAsync(final_state + b * nst, dfin, lo.st, cudaMemcpyDeviceToHost, pl->d2h);
    if (e == cudaSuccess) e = cudaEventRecord(pl->out_done[kb], pl->d2h);
    if (e != cudaSuccess) s = cuda_status(e);
  }
  // join: the caller's stream continues after both copy streams (also after a
  // failure, so that neither is left forked from a capture)
  cudaError_t ej = cudaEventRecord(pl->join, pl->d2h);
  if (ej == cudaSuccess) ej = cudaStreamWaitEvent(st, pl->join, 0);
  if (ej == cudaSuccess) ej = cudaEventRecord(pl->join, pl->h2d);
  if (ej == cudaSuccess) ej = cudaStreamWaitEvent(st, pl->join, 0);
  if (ej != cudaSuccess && s == SSD_OK) s = cuda_status(ej);
  return s;
}

}  // extern "C"
