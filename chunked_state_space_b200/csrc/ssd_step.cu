// Recurrent (decode) step: one token per call with the state carried in
// place -- the token recurrence of "分块推理：解锁循环模型并行计算，实现长序列高效处理" §2
// (h_t = a_t h_{t-1} + B_t x_t^T, y_t = C_t^T h_t, here with the skip D x_t;
// with SSD_FLAG_INPUT_DT the input term is dt_t B_t x_t^T),
// the mode a model runs in when it generates with a state cache.
//
// HBM-bound on the fp32 state: every call reads and writes N*P*4 bytes per
// (batch, head).  One block per (batch, head).  The staged kernel (P % 4 ==
// 0, N <= 128, 16-byte aligned state) copies the block's state tile into
// shared memory with one bulk copy and updates it from there (below); the
// scalar kernel covers every other shape.  a = exp(dt A) is evaluated once per
// warp and broadcast.  y is reduced over the state rows in shared memory in a
// fixed order (deterministic).
#include "ssd_common.cuh"
#include "umma.cuh"

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

// Staged form (P % 4 == 0, N <= 128, state 16-byte aligned): thread 0 brings
// the block's whole state tile [N][P] f32 (at most 32 KB) into shared memory
// with one bulk copy while the others load B, C, dt, A and x; the 256 threads
// then update the tile from shared memory and write it back with 128-bit
// stores.  A block holds 37 KB of shared memory and few registers, so six run
// per SM and the whole state of a 2.7B-shaped layer is in flight at once.
template <typename T>
__global__ void __launch_bounds__(256) k_ssd_step_bulk(const T* __restrict__ x, const float* __restrict__ dt,
                                                       const float* __restrict__ A, const T* __restrict__ Bm,
                                                       const T* __restrict__ Cm, const float* __restrict__ D,
                                                       float* __restrict__ state, T* __restrict__ y, int H, int G,
                                                       int N, int P, int input_dt) {
  using namespace umma;
  extern __shared__ __align__(128) float tile[];  // [N][P]
  __shared__ float4 part[256];
  __shared__ float sb[128], sc[128];  // B and C of the token, one entry per state row
  __shared__ __align__(8) uint64_t bar;
  const int bh = blockIdx.x;
  const int b = bh / H, h = bh % H;
  const int g = h / (H / G);
  const int C4 = P / 4, R = 256 / C4;
  const int tid = threadIdx.x, lane = tid & 31;
  const int c = tid % C4, r = tid / C4;
  float* st = state + (int64_t)bh * N * P;
  const uint32_t bytes = (uint32_t)(N * P) * 4u;
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&bar, bytes);
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(tile)),
        "l"(st), "r"(bytes), "r"(smem_u32(&bar))
        : "memory");
  }
  const T* bg = Bm + ((int64_t)b * G + g) * N;
  const T* cg = Cm + ((int64_t)b * G + g) * N;
  float bt = 0.f, ct = 0.f;
  if (tid < N) {
    bt = to_f32(bg[tid]);
    ct = to_f32(cg[tid]);
  }
  const float dtv = dt[bh];
  const float Ah = lane == 0 ? A[h] : 0.f;
  float xp[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) xp[i] = to_f32(x[(int64_t)bh * P + 4 * c + i]);
  float a = 0.f;
  if (lane == 0) a = expf(dtv * Ah);
  a = __shfl_sync(0xffffffffu, a, 0);
  float xin[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) xin[i] = input_dt ? dtv * xp[i] : xp[i];
  if (tid < N) {
    sb[tid] = bt;
    sc[tid] = ct;
  }
  __syncthreads();  // sb, sc and the initialised barrier are visible to all
  if (!mbar_wait(&bar, 0)) {  // bounded: the copy of valid memory lands unless the device is wedged
    if (tid == 0) atomicExch(&g_device_status, 2);
    return;
  }
  const float4* t4 = reinterpret_cast<const float4*>(tile);
  float4* st4 = reinterpret_cast<float4*>(st);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (r < R) {
    for (int n = r; n < N; n += R) {
      const float4 v = t4[n * C4 + c];
      const float bn = sb[n], cn = sc[n];
      float4 o;
      o.x = fmaf(a, v.x, bn * xin[0]);
      o.y = fmaf(a, v.y, bn * xin[1]);
      o.z = fmaf(a, v.z, bn * xin[2]);
      o.w = fmaf(a, v.w, bn * xin[3]);
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
    y[(int64_t)bh * P + tid] = from_f32<T>(s + d * to_f32(x[(int64_t)bh * P + tid]));
  }
}

cudaError_t launch_ssd_step(const Problem& p, float* state, cudaStream_t st) {
  const int P = (int)p.P;
  if (P % 4 == 0 && (reinterpret_cast<uintptr_t>(state) & 15u) == 0 && p.N <= 128) {
    const int threads = 256;  // (P/4) columns x (1024/P) rows per pass
    const size_t tile = sizeof(float) * (size_t)p.N * P;  // <= 32 KB
    if (p.io == SSD_BF16)
      k_ssd_step_bulk<__nv_bfloat16><<<(unsigned)(p.B * p.H), threads, tile, st>>>(
          (const __nv_bfloat16*)p.x, p.dt, p.A, (const __nv_bfloat16*)p.Bm, (const __nv_bfloat16*)p.Cm, p.D, state,
          (__nv_bfloat16*)p.y, (int)p.H, (int)p.G, (int)p.N, P, p.input_dt);
    else
      k_ssd_step_bulk<float><<<(unsigned)(p.B * p.H), threads, tile, st>>>(
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
