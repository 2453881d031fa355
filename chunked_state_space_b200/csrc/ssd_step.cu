// Recurrent (decode) step: one token per call with the state carried in
// place -- the token recurrence of "分块推理：解锁循环模型并行计算，实现长序列高效处理" §2
// (h_t = a_t h_{t-1} + B_t x_t^T, y_t = C_t^T h_t, here with the skip D x_t;
// with SSD_FLAG_INPUT_DT the input term is dt_t B_t x_t^T),
// the mode a model runs in when it generates with a state cache.
//
// HBM-bound on the fp32 state: every call reads and writes N*P*4 bytes per
// (batch, head).  One block per (batch, head).  The vector kernel (P % 4 == 0,
// 16-byte aligned state) gives thread (c, r) the four columns 4c..4c+3 of
// state rows r, r + R, ... (R = 256 / (P/4)): 128-bit loads and stores, all
// of a thread's rows loaded before any is written back, so a block keeps its
// whole 32 KB state tile in flight.  The scalar kernel covers every other
// shape.  a = exp(dt A) is evaluated once per warp and broadcast.  y is
// reduced over r in shared memory in a fixed order (deterministic).
#include "ssd_common.cuh"

namespace ssd {

template <typename T>
__global__ void __launch_bounds__(256) k_ssd_step(const T* __restrict__ x, const float* __restrict__ dt,
                                                  const float* __restrict__ A, const T* __restrict__ Bm,
                                                  const T* __restrict__ Cm, const float* __restrict__ D,
                                                  float* __restrict__ state, T* __restrict__ y, int H, int G, int N,
                                                  int P, int input_dt) {
  __shared__ float part[256];
  const int bh = blockIdx.x;
  const int b = bh / H, h = bh % H;
  const int g = h / (H / G);
  const int R = blockDim.x / P;
  const int tid = threadIdx.x;
  const int p = tid % P, r = tid / P;
  const bool on = r < R;
  const float a = expf(dt[bh] * A[h]);
  const float xp = to_f32(x[(int64_t)bh * P + p]);
  const float xin = input_dt ? dt[bh] * xp : xp;  // the input term's x (the skip uses xp)
  const T* bg = Bm + ((int64_t)b * G + g) * N;
  const T* cg = Cm + ((int64_t)b * G + g) * N;
  float* st = state + (int64_t)bh * N * P;
  float acc = 0.f;
  if (on) {
    for (int n = r; n < N; n += R) {
      float* e = st + (int64_t)n * P + p;
      const float v = fmaf(a, *e, to_f32(bg[n]) * xin);
      *e = v;
      acc = fmaf(to_f32(cg[n]), v, acc);
    }
  }
  part[tid] = on ? acc : 0.f;
  __syncthreads();
  if (tid < P) {
    float s = 0.f;
    for (int k = 0; k < R; ++k) s += part[k * P + tid];
    const float d = D ? D[h] : 0.f;
    y[(int64_t)bh * P + tid] = from_f32<T>(s + d * xp);
  }
}

// 128-bit form: P % 4 == 0, state 16-byte aligned, N <= 128.  Thread (c, r):
// columns 4c..4c+3, rows r + R k for k < N / R (R = 4 * 256 / P rows per pass).
template <typename T>
__global__ void __launch_bounds__(256) k_ssd_step_v4(const T* __restrict__ x, const float* __restrict__ dt,
                                                     const float* __restrict__ A, const T* __restrict__ Bm,
                                                     const T* __restrict__ Cm, const float* __restrict__ D,
                                                     float* __restrict__ state, T* __restrict__ y, int H, int G, int N,
                                                     int P, int input_dt) {
  __shared__ float4 part[256];
  constexpr int kMaxRows = 16;  // N <= 128 rows over at least R = 16 rows per pass (P <= 64)
  const int bh = blockIdx.x;
  const int b = bh / H, h = bh % H;
  const int g = h / (H / G);
  const int C4 = P / 4, R = 256 / C4;
  const int tid = threadIdx.x, lane = tid & 31;
  const int c = tid % C4, r = tid / C4;
  const float dtv = dt[bh];
  float a = 0.f;
  if (lane == 0) a = expf(dtv * A[h]);
  a = __shfl_sync(0xffffffffu, a, 0);
  float xp[4], xin[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    xp[i] = to_f32(x[(int64_t)bh * P + 4 * c + i]);
    xin[i] = input_dt ? dtv * xp[i] : xp[i];
  }
  const T* bg = Bm + ((int64_t)b * G + g) * N;
  const T* cg = Cm + ((int64_t)b * G + g) * N;
  float4* st4 = reinterpret_cast<float4*>(state + (int64_t)bh * N * P);
  float4 v[kMaxRows];
  // rows of this thread; threads past the last full pass (r >= R, when C4
  // does not divide 256) own none
  const int nk = r < R ? (N - r + R - 1) / R : 0;
#pragma unroll
  for (int k = 0; k < kMaxRows; ++k)
    if (k < nk) v[k] = st4[(int64_t)(r + k * R) * C4 + c];
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int k = 0; k < kMaxRows; ++k) {
    if (k < nk) {
      const int n = r + k * R;
      const float bn = to_f32(bg[n]), cn = to_f32(cg[n]);
      float4 o;
      o.x = fmaf(a, v[k].x, bn * xin[0]);
      o.y = fmaf(a, v[k].y, bn * xin[1]);
      o.z = fmaf(a, v[k].z, bn * xin[2]);
      o.w = fmaf(a, v[k].w, bn * xin[3]);
      st4[(int64_t)n * C4 + c] = o;
      acc.x = fmaf(cn, o.x, acc.x);
      acc.y = fmaf(cn, o.y, acc.y);
      acc.z = fmaf(cn, o.z, acc.z);
      acc.w = fmaf(cn, o.w, acc.w);
    }
  }
  part[tid] = acc;
  __syncthreads();
  if (tid < P) {
    const int cc = tid / 4, i = tid % 4;
    float s = 0.f;
    for (int k = 0; k < R; ++k) {
      const float4 q = part[k * C4 + cc];
      s += (i == 0) ? q.x : (i == 1) ? q.y : (i == 2) ? q.z : q.w;
    }
    const float d = D ? D[h] : 0.f;
    const float xv = to_f32(x[(int64_t)bh * P + tid]);
    y[(int64_t)bh * P + tid] = from_f32<T>(s + d * xv);
  }
}

cudaError_t launch_ssd_step(const Problem& p, float* state, cudaStream_t st) {
  const int P = (int)p.P;
  if (P % 4 == 0 && (reinterpret_cast<uintptr_t>(state) & 15u) == 0 && p.N <= 128) {
    const int threads = 256;  // (P/4) columns x (1024/P) rows per pass
    if (p.io == SSD_BF16)
      k_ssd_step_v4<__nv_bfloat16><<<(unsigned)(p.B * p.H), threads, 0, st>>>(
          (const __nv_bfloat16*)p.x, p.dt, p.A, (const __nv_bfloat16*)p.Bm, (const __nv_bfloat16*)p.Cm, p.D, state,
          (__nv_bfloat16*)p.y, (int)p.H, (int)p.G, (int)p.N, P, p.input_dt);
    else
      k_ssd_step_v4<float><<<(unsigned)(p.B * p.H), threads, 0, st>>>(
          (const float*)p.x, p.dt, p.A, (const float*)p.Bm, (const float*)p.Cm, p.D, state, (float*)p.y, (int)p.H,
          (int)p.G, (int)p.N, P, p.input_dt);
    return cudaGetLastError();
  }
  const int threads = (256 / P) * P;
  if (p.io == SSD_BF16)
    k_ssd_step<__nv_bfloat16><<<(unsigned)(p.B * p.H), threads, 0, st>>>(
        (const __nv_bfloat16*)p.x, p.dt, p.A, (const __nv_bfloat16*)p.Bm, (const __nv_bfloat16*)p.Cm, p.D, state,
        (__nv_bfloat16*)p.y, (int)p.H, (int)p.G, (int)p.N, P, p.input_dt);
  else
    k_ssd_step<float><<<(unsigned)(p.B * p.H), threads, 0, st>>>((const float*)p.x, p.dt, p.A, (const float*)p.Bm,
                                                                 (const float*)p.Cm, p.D, state, (float*)p.y,
                                                                 (int)p.H, (int)p.G, (int)p.N, P, p.input_dt);
  return cudaGetLastError();
}

}  // namespace ssd
