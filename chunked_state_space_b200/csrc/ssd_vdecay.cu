// The scan with a vector-valued decay, one rate per state channel n: the
// diagonal state matrix of the selective scan ("告别Transformer的二次方噩梦…"
// §2.1) and the per-channel decays of the recurrences "分块推理…" §6 names
// (RWKV, xLSTM).  For every (batch, head):
//   a_t[n] = exp(dt[b,t,h] Av[h,n])
//   h_t[n,:] = a_t[n] h_{t-1}[n,:] + B[b,t,g,n] x[b,t,h,:]
//   y_t = C[b,t,g,:]^T h_t + D[h] x[b,t,h,:]
// With channel-dependent decays the chunked form's intra-chunk term no longer
// factors into (C B^T) (.) L, so this path runs the token recurrence itself on
// CUDA cores (fp32 state, fp32 or bf16 io): one block per (batch, head), tiles
// of 16 tokens staged in shared memory (decays, B, C, x), thread (p, g) owning
// column p of state rows g, g + R, ... (R = 256 / P rows per pass) in
// registers, and y reduced over the R row groups in a fixed order.  P = 64
// with N % 16 == 0 takes a vectorised form of the same kernel.
#include "ssd_common.cuh"

namespace ssd {

namespace vdecay {
constexpr int TT = 16;          // tokens per staged tile
constexpr int THREADS = 256;
constexpr int MAXN = 128, MAXP = 64;
constexpr int MAXK = 32;        // state rows per thread: N <= 128 rows over R >= 4 groups
}  // namespace vdecay

template <typename T>
__global__ void __launch_bounds__(vdecay::THREADS) k_ssd_scan_vdecay(
    const T* __restrict__ x, const float* __restrict__ dt, const float* __restrict__ Av, const T* __restrict__ Bm,
    const T* __restrict__ Cm, const float* __restrict__ D, const float* __restrict__ init, T* __restrict__ y,
    float* __restrict__ final_state, int64_t L, int H, int G, int N, int P) {
  using namespace vdecay;
  __shared__ float s_a[TT][MAXN], s_b[TT][MAXN], s_c[TT][MAXN], s_x[TT][MAXP];
  __shared__ float s_y[TT][THREADS];  // [token][row group * P + p]
  const int bh = blockIdx.x;
  const int b = bh / H, h = bh % H, g = h / (H / G);
  const int tid = threadIdx.x;
  const int R = THREADS / P;          // row groups
  const int p = tid % P, rg = tid / P;
  const bool on = rg < R;             // threads past the last full group own nothing
  float st[MAXK];
  const int nk = on ? (N - rg + R - 1) / R : 0;
  const float* ini = init ? init + (int64_t)bh * N * P : nullptr;
#pragma unroll
  for (int k = 0; k < MAXK; ++k) st[k] = (k < nk && ini) ? ini[(int64_t)(rg + k * R) * P + p] : 0.f;
  const float Dh = D ? D[h] : 0.f;
  const float* avh = Av + (int64_t)h * N;
  for (int64_t t0 = 0; t0 < L; t0 += TT) {
    // stage the tile: decays a_t[n], B_t[n], C_t[n], x_t[p] (past L: a = 1, rest 0)
    for (int i = tid; i < TT * N; i += THREADS) {
      const int tt = i / N, n = i % N;
      const int64_t t = t0 + tt;
      const bool in = t < L;
      const int64_t bc = ((int64_t)(b * L + (in ? t : 0)) * G + g) * N + n;
      s_a[tt][n] = in ? expf(dt[(int64_t)(b * L + t) * H + h] * avh[n]) : 1.f;
      s_b[tt][n] = in ? to_f32(Bm[bc]) : 0.f;
      s_c[tt][n] = in ? to_f32(Cm[bc]) : 0.f;
    }
    for (int i = tid; i < TT * P; i += THREADS) {
      const int tt = i / P, pp = i % P;
      const int64_t t = t0 + tt;
      s_x[tt][pp] = t < L ? to_f32(x[((int64_t)(b * L + t) * H + h) * P + pp]) : 0.f;
    }
    __syncthreads();
    // the recurrence over the tile's tokens, this thread's state entries
#pragma unroll 1
    for (int tt = 0; tt < TT; ++tt) {
      const float xv = s_x[tt][p];
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < MAXK; ++k) {
        if (k < nk) {
          const int n = rg + k * R;
          st[k] = fmaf(s_a[tt][n], st[k], s_b[tt][n] * xv);
          acc = fmaf(s_c[tt][n], st[k], acc);
        }
      }
      s_y[tt][tid] = on ? acc : 0.f;
    }
    __syncthreads();
    // y_t[p] = sum over row groups (fixed order) + D x_t[p]
    for (int i = tid; i < TT * P; i += THREADS) {
      const int tt = i / P, pp = i % P;
      const int64_t t = t0 + tt;
      if (t < L) {
        float s = 0.f;
        for (int r = 0; r < R; ++r) s += s_y[tt][r * P + pp];
        y[((int64_t)(b * L + t) * H + h) * P + pp] = from_f32<T>(s + Dh * s_x[tt][pp]);
      }
    }
    __syncthreads();  // the next tile overwrites the staging buffers
  }
  if (final_state) {
    float* fo = final_state + (int64_t)bh * N * P;
#pragma unroll
    for (int k = 0; k < MAXK; ++k)
      if (k < nk) fo[(int64_t)(rg + k * R) * P + p] = st[k];
  }
}

namespace vdecay {
// Two fp32 lanes per instruction (sm_100 packed f32x2), each rounded like
// the scalar operation.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 c;
  asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rc, ra, rb;\n\t"
      "mov.b64 {%0, %1}, rc;\n\t}"
      : "=f"(c.x), "=f"(c.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return c;
}
constexpr int VP = 64;                 // head dim of the vectorised kernel
constexpr int VR = THREADS / VP;       // 4 row groups
constexpr int VK = MAXN / VR;          // at most 32 state rows per thread
constexpr int VTT = 8;                 // tokens per staged tile (its loads are prefetched into registers)
}  // namespace vdecay

// The same recurrence for P = 64 and N % 16 == 0 (the model shapes): thread
// (p, g) owns state rows g, g + 4, ..., and the staged decays, B and C are laid
// out [token][g][k] so that one 128-bit shared-memory load (a broadcast: the
// warp's 32 threads share g) brings four of its rows, and the updates run on
// packed fp32x2 instructions.  Same arithmetic per state entry as above
// (h = fma(a, h, b x)); y sums its rows in four interleaved partial sums.
// Tiles of 8 tokens, the next tile's loads in registers while this one is
// computed; 120 registers, two blocks per SM.
template <typename T>
__global__ void __launch_bounds__(vdecay::THREADS, 2) k_ssd_scan_vdecay64(
    const T* __restrict__ x, const float* __restrict__ dt, const float* __restrict__ Av, const T* __restrict__ Bm,
    const T* __restrict__ Cm, const float* __restrict__ D, const float* __restrict__ init, T* __restrict__ y,
    float* __restrict__ final_state, int64_t L, int H, int G, int N) {
  using namespace vdecay;
  constexpr int MM = VTT * MAXN / THREADS;  // staged (token, row) entries per thread
  constexpr int MX = VTT * VP / THREADS;    // staged x entries per thread
  __shared__ __align__(16) float s_a[VTT][MAXN], s_b[VTT][MAXN], s_c[VTT][MAXN];  // [tt][g * nk + k]
  __shared__ float s_x[VTT][VP];
  __shared__ float s_y[VTT][THREADS];
  const int bh = blockIdx.x;
  const int b = bh / H, h = bh % H, g = h / (H / G);
  const int tid = threadIdx.x;
  const int p = tid % VP, rg = tid / VP;
  const int nk = N / VR;  // rows per thread, a multiple of 4
  float st[VK];
  const float* ini = init ? init + (int64_t)bh * N * VP : nullptr;
#pragma unroll
  for (int k = 0; k < VK; ++k) st[k] = (k < nk && ini) ? ini[(int64_t)(rg + k * VR) * VP + p] : 0.f;
  const float Dh = D ? D[h] : 0.f;
  const float* avh = Av + (int64_t)h * N;
  // The next tile's dt, B, C and x are loaded into registers while this tile
  // is computed, and written to shared memory (decays formed) after it.
  float pdt[MM];
  T pb[MM], pc[MM], px[MX];
  auto fetch = [&](int64_t t0) {
#pragma unroll
    for (int m = 0; m < MM; ++m) {
      const int i = tid + m * THREADS;
      const int tt = i / N, n = i % N;
      const int64_t t = t0 + tt;
      const bool in = i < VTT * N && t < L;
      const int64_t bc = ((int64_t)(b * L + (in ? t : 0)) * G + g) * N + n;
      pdt[m] = in ? dt[(int64_t)(b * L + t) * H + h] : 0.f;
      pb[m] = in ? Bm[bc] : from_f32<T>(0.f);
      pc[m] = in ? Cm[bc] : from_f32<T>(0.f);
    }
#pragma unroll
    for (int m = 0; m < MX; ++m) {
      const int i = tid + m * THREADS;
      const int tt = i / VP, pp = i % VP;
      const int64_t t = t0 + tt;
      px[m] = t < L ? x[((int64_t)(b * L + t) * H + h) * VP + pp] : from_f32<T>(0.f);
    }
  };
  // row n = g + k * 4 of token tt goes to [tt][g * nk + k]; past L: a = 1, b = c = x = 0
  auto stage = [&](int64_t t0) {
#pragma unroll
    for (int m = 0; m < MM; ++m) {
      const int i = tid + m * THREADS;
      if (i < VTT * N) {
        const int tt = i / N, n = i % N;
        const int j = (n % VR) * nk + n / VR;
        const bool in = t0 + tt < L;
        s_a[tt][j] = in ? expf(pdt[m] * avh[n]) : 1.f;
        s_b[tt][j] = to_f32(pb[m]);
        s_c[tt][j] = to_f32(pc[m]);
      }
    }
#pragma unroll
    for (int m = 0; m < MX; ++m) {
      const int i = tid + m * THREADS;
      s_x[i / VP][i % VP] = to_f32(px[m]);
    }
  };
  fetch(0);
  for (int64_t t0 = 0; t0 < L; t0 += VTT) {
    stage(t0);
    __syncthreads();
    if (t0 + VTT < L) fetch(t0 + VTT);
#pragma unroll 1
    for (int tt = 0; tt < VTT; ++tt) {
      const float xv = s_x[tt][p];
      const float2 x2 = make_float2(xv, xv);
      const float4* a4 = reinterpret_cast<const float4*>(&s_a[tt][rg * nk]);
      const float4* b4 = reinterpret_cast<const float4*>(&s_b[tt][rg * nk]);
      const float4* c4 = reinterpret_cast<const float4*>(&s_c[tt][rg * nk]);
      // y partial sums in four lanes (rows k = 0, 1, 2, 3 mod 4), added at the end
      float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
      for (int q = 0; q < VK / 4; ++q) {
        if (4 * q < nk) {
          const float4 a = a4[q], bb = b4[q], c = c4[q];
          const float2 bx0 = mul2(make_float2(bb.x, bb.y), x2), bx1 = mul2(make_float2(bb.z, bb.w), x2);
          const float2 h0 = fma2(make_float2(a.x, a.y), make_float2(st[4 * q], st[4 * q + 1]), bx0);
          const float2 h1 = fma2(make_float2(a.z, a.w), make_float2(st[4 * q + 2], st[4 * q + 3]), bx1);
          st[4 * q] = h0.x;
          st[4 * q + 1] = h0.y;
          st[4 * q + 2] = h1.x;
          st[4 * q + 3] = h1.y;
          acc0 = fma2(make_float2(c.x, c.y), h0, acc0);
          acc1 = fma2(make_float2(c.z, c.w), h1, acc1);
        }
      }
      s_y[tt][tid] = (acc0.x + acc0.y) + (acc1.x + acc1.y);
    }
    __syncthreads();
    for (int i = tid; i < VTT * VP; i += THREADS) {
      const int tt = i / VP, pp = i % VP;
      const int64_t t = t0 + tt;
      if (t < L) {
        float s = 0.f;
        for (int r = 0; r < VR; ++r) s += s_y[tt][r * VP + pp];
        y[((int64_t)(b * L + t) * H + h) * VP + pp] = from_f32<T>(s + Dh * s_x[tt][pp]);
      }
    }
    __syncthreads();  // the next tile is staged over this one
  }
  if (final_state) {
    float* fo = final_state + (int64_t)bh * N * VP;
#pragma unroll
    for (int k = 0; k < VK; ++k)
      if (k < nk) fo[(int64_t)(rg + k * VR) * VP + p] = st[k];
  }
}

cudaError_t launch_scan_vdecay(const Problem& p, const float* Av, const float* init, float* final_state,
                               cudaStream_t st) {
  using namespace vdecay;
  if (p.N > MAXN || p.P > MAXP || p.P < 1) return cudaErrorInvalidValue;
  const unsigned grid = (unsigned)(p.B * p.H);
  if (p.P == VP && p.N % 16 == 0) {
    if (p.io == SSD_BF16)
      k_ssd_scan_vdecay64<__nv_bfloat16><<<grid, THREADS, 0, st>>>(
          (const __nv_bfloat16*)p.x, p.dt, Av, (const __nv_bfloat16*)p.Bm, (const __nv_bfloat16*)p.Cm, p.D, init,
          (__nv_bfloat16*)p.y, final_state, p.L, (int)p.H, (int)p.G, (int)p.N);
    else
      k_ssd_scan_vdecay64<float><<<grid, THREADS, 0, st>>>((const float*)p.x, p.dt, Av, (const float*)p.Bm,
                                                            (const float*)p.Cm, p.D, init, (float*)p.y, final_state,
                                                            p.L, (int)p.H, (int)p.G, (int)p.N);
    return cudaGetLastError();
  }
  if (p.io == SSD_BF16)
    k_ssd_scan_vdecay<__nv_bfloat16><<<grid, THREADS, 0, st>>>(
        (const __nv_bfloat16*)p.x, p.dt, Av, (const __nv_bfloat16*)p.Bm, (const __nv_bfloat16*)p.Cm, p.D, init,
        (__nv_bfloat16*)p.y, final_state, p.L, (int)p.H, (int)p.G, (int)p.N, (int)p.P);
  else
    k_ssd_scan_vdecay<float><<<grid, THREADS, 0, st>>>((const float*)p.x, p.dt, Av, (const float*)p.Bm,
                                                        (const float*)p.Cm, p.D, init, (float*)p.y, final_state,
                                                        p.L, (int)p.H, (int)p.G, (int)p.N, (int)p.P);
  return cudaGetLastError();
}

}  // namespace ssd

// Entry point (validation as the other scans; no workspace).
extern "C" ssd_status ssd_scan_fwd_vdecay(const ssd_dims* d, const void* x, const float* dt, const float* Av,
                                          const void* Bm, const void* Cm, const float* D, const float* init_state,
                                          void* y, float* final_state, void* stream) {
  using namespace ssd;
  ssd_status s = validate_dims(d);
  if (s != SSD_OK) return s;
  if (d->flags != 0) return SSD_ERR_UNSUPPORTED;
  if (!Av) return SSD_ERR_INVALID_ARG;
  // A here is the [H] slot of the common checks; Av [H, N] is checked on its own
  s = validate_scan_args(d, x, dt, Av, Bm, Cm, D, init_state, y, final_state, /*natural_alignment=*/true);
  if (s != SSD_OK) return s;
  const size_t es = d->io_dtype == SSD_BF16 ? 2 : 4;
  const uintptr_t ylo = reinterpret_cast<uintptr_t>(y);
  const uintptr_t yhi = ylo + es * (size_t)d->batch * d->seqlen * d->nheads * d->headdim;
  const uintptr_t alo = reinterpret_cast<uintptr_t>(Av), ahi = alo + sizeof(float) * (size_t)d->nheads * d->dstate;
  if (alo < yhi && ylo < ahi) return SSD_ERR_INVALID_ARG;
  Problem p = make_problem(d);
  p.x = x; p.dt = dt; p.Bm = Bm; p.Cm = Cm; p.D = D; p.y = y;
  return cuda_status(launch_scan_vdecay(p, Av, init_state, final_state, static_cast<cudaStream_t>(stream)));
}
