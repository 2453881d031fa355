// Recurrent (decode) step: one token per call with the state carried in
// place -- the token recurrence of "分块推理：解锁循环模型并行计算，实现长序列高效处理" §2
// (h_t = a_t h_{t-1} + B_t x_t^T, y_t = C_t^T h_t, here with the skip D x_t;
// with SSD_FLAG_INPUT_DT the input term is dt_t B_t x_t^T),
// the mode a model runs in when it generates with a state cache.
//
// HBM-bound on the fp32 state: every call reads and writes N*P*4 bytes per
// (batch, head).  One block per (batch, head); thread (p, r) owns column p of
// the state rows r, r + R, r + 2R, ... (R = blockDim / P), so warps read and
// write contiguous row segments; y is reduced over r in shared memory in a
// fixed order (deterministic).
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

cudaError_t launch_ssd_step(const Problem& p, float* state, cudaStream_t st) {
  const int P = (int)p.P;
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
