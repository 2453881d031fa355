// Split schedule shared by the fused scan kernels: the sequences (units) of a
// launch are concatenated into one list of 128-token sub-chunks and cut into
// equal ranges, one per persistent CTA.  When there are at least as many
// units as CTAs, a range is at least one unit long, so it holds at most a
// tail piece of one unit, whole units, and a head piece of the next.  The CTA
// runs its head piece first and publishes that piece's end state (the carry:
// the page's inter-chunk recursion handed across CTAs, "分块推理…" §2.2) to a
// workspace slot with a release flag; the next CTA needs it only for its tail
// piece, which it runs last.  With one unit per CTA this is the plain
// one-sequence-per-CTA launch.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {
namespace split {

// The sub-chunks of CTA c: [lo, hi) of the concatenated list, run in the order
// head piece of the last sequence (if the range ends inside it), whole
// sequences, tail piece of the first sequence (if the range starts inside it).
struct Range {
  int64_t lo, hi;
  int nsub;
  int64_t u_lo, u_hi;  // first and last sequence touched
  int j_lo, j_hi;      // start of the first piece, end (exclusive) of the last piece
  int head_len;        // sub-chunks of the leading head piece (0 if none)
  int tail_len;        // sub-chunks of the trailing tail piece (0 if none)
  int64_t full_first;  // first whole sequence
  __device__ void init(int64_t total, int nctas, int c, int ns) {
    nsub = ns;
    lo = total * c / nctas;
    hi = total * (c + 1) / nctas;
    u_lo = lo / ns;
    j_lo = (int)(lo % ns);
    u_hi = (hi - 1) / ns;
    j_hi = (int)((hi - 1) % ns) + 1;
    head_len = (u_hi > u_lo && j_hi < ns) ? j_hi : 0;
    tail_len = j_lo > 0 ? ns - j_lo : 0;
    full_first = j_lo > 0 ? u_lo + 1 : u_lo;
  }
  __device__ int64_t count() const { return hi - lo; }
  // sequence, sub-chunk, and piece boundaries of the k-th sub-chunk this CTA runs
  __device__ void at(int64_t k, int64_t& u, int& j, bool& first, bool& last, bool& carry_in,
                     bool& carry_out) const {
    if (k < head_len) {
      u = u_hi;
      j = (int)k;
      first = (k == 0);
      last = (k == head_len - 1);
      carry_in = false;
      carry_out = last;
      return;
    }
    const int64_t kk = k - head_len;
    const int64_t nfull_sub = count() - head_len - tail_len;
    if (kk < nfull_sub) {
      u = full_first + kk / nsub;
      j = (int)(kk % nsub);
      first = (j == 0);
      last = (j == nsub - 1);
      carry_in = carry_out = false;
      return;
    }
    const int64_t kt = kk - nfull_sub;
    u = u_lo;
    j = j_lo + (int)kt;
    first = (kt == 0);
    last = (j == nsub - 1);
    carry_in = first;
    carry_out = false;
  }
};

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Streaming multiprocessors of the current device (queried once per device).
inline int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

// CTAs of a split launch over `units` sequences: one per SM, never more than
// the units (so no range lies strictly inside one unit).
inline int ctas(int64_t units) {
  const int64_t n = sm_count();
  return (int)(units < n ? units : n);
}

// Workspace of a split launch: `slot_floats` per CTA for the carry, then one
// int flag per CTA (zeroed before every launch); 0 when every CTA runs whole
// units anyway.
inline size_t workspace_bytes(int64_t units, size_t slot_floats) {
  const int n = ctas(units);
  if (n >= units) return 0;
  return (size_t)n * slot_floats * sizeof(float) + (size_t)((n * sizeof(int) + 255) / 256 * 256);
}

}  // namespace split
}  // namespace ssd
