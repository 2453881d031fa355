// Segment-round schedule of the persistent fused scan kernels.  Every
// sequence (unit) of the launch is cut into nseg equal segments of
// seg = nsub / nseg 128-token sub-chunks; the (segment r, sequence q) work
// items are numbered segment-major, v = r * nseq + q, and persistent CTA c
// runs the items c, c + G, c + 2G, ... in that order (G CTAs, one per SM).
// A segment after the first starts from the end state of the segment before
// it: the page's inter-chunk recursion ("分块推理…" §2.2: b(c) from b(c-1))
// handed across CTAs through a workspace slot per sequence and a flag that
// counts the segments of the sequence whose end state has been published.
// With nseq >= G the item a segment waits for (v - nseq) lies at least one
// round earlier, so in the steady state the carry is there when it is needed.
// Numbering the items segment-major keeps the CTAs of one round on the same
// segment of neighbouring sequences: the heads of one batch then walk the
// same tokens together and read each B/C tile from DRAM once, the rest from
// L2.  With nseg = 1 the schedule runs whole sequences, round-robin.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {
namespace split {

struct Rounds {
  int64_t nseq;   // sequences of the launch
  int nseg, seg;  // segments per sequence, sub-chunks per segment
  int G, c;       // CTAs of the launch, this CTA
  int64_t items;  // work items of this CTA
  __device__ void init(int64_t nseq_, int nsub, int nseg_, int G_, int c_) {
    nseq = nseq_;
    nseg = nseg_;
    seg = nsub / nseg_;
    G = G_;
    c = c_;
    const int64_t all = nseq * nseg;
    items = all > c ? (all - c + G - 1) / G : 0;
  }
  __device__ int64_t count() const { return items * seg; }
  // sequence u, sub-chunk j, segment r, and segment boundaries of the k-th
  // sub-chunk this CTA runs
  __device__ void at(int64_t k, int64_t& u, int& j, int& r, bool& first, bool& last, bool& carry_in,
                     bool& carry_out) const {
    const int64_t i = k / seg;
    const int o = (int)(k - i * seg);
    const int64_t v = c + i * G;
    r = (int)(v / nseq);
    u = v - (int64_t)r * nseq;
    j = r * seg + o;
    first = (o == 0);
    last = (o == seg - 1);
    carry_in = first && r > 0;
    carry_out = last && r < nseg - 1;
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

// Segments per sequence for `nseq` sequences of `nsub` sub-chunks on G CTAs:
// the divisor of nsub that minimises rounds x (segment length + the carry's
// cost, about one and a half sub-chunks of traffic), among those that keep
// every carry at least one round back (nseq >= G); 1 otherwise.
inline int segments(int64_t nseq, int nsub, int G) {
  if (nseq < G || nsub <= 1) return 1;
  int best = 1;
  double best_cost = 0;
  for (int n = 1; n <= nsub; ++n) {
    if (nsub % n) continue;
    const int64_t rounds = (nseq * n + G - 1) / G;
    const double cost = (double)rounds * ((double)(nsub / n) + (n > 1 ? 1.5 : 0.0));
    if (n == 1 || cost < best_cost) {
      best = n;
      best_cost = cost;
    }
  }
  return best;
}

// Workspace of a segmented launch: one carry slot of `slot_floats` per
// sequence, then one int flag per sequence (zeroed before every launch); 0
// when the sequences run whole.
inline size_t workspace_bytes(int64_t nseq, int nseg, size_t slot_floats) {
  if (nseg <= 1) return 0;
  return (size_t)nseq * slot_floats * sizeof(float) + (size_t)((nseq * sizeof(int) + 255) / 256 * 256);
}

}  // namespace split
}  // namespace ssd
