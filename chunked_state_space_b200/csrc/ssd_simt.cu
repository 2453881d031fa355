// CUDA-core kernels of the chunked SSD scan: the four steps of
// "分块推理：解锁循环模型并行计算，实现长序列高效处理" §2.1-§2.2 in fp32 arithmetic, for
// fp32 or bf16 io, plus the layer-to-layer RMS normalisation.  This is the
// exact path (fp32 io is checked at 1e-5) and the fallback for sizes the
// tensor-core kernels do not cover.
#include <type_traits>

#include "ssd_common.cuh"

namespace ssd {

// ---------------------------------------------------------------------------
// Step 1: lam[b,h,c,i] = sum_{r<=i} dt[b,cQ+r,h] * A[h], summed sequentially so
// that a difference lam[t] - lam[s] only carries the rounding of the t - s
// additions between them.  grid (nc, B, ceil(H/32)), block 32, smem [Q][33].
__global__ void k_chunk_cumsum(const float* __restrict__ dt, int64_t sdt, const float* __restrict__ A,
                               float* __restrict__ lam, int64_t L, int H, int Q, int nc) {
  extern __shared__ float sm[];
  const int c = blockIdx.x, b = blockIdx.y, h0 = blockIdx.z * 32, lane = threadIdx.x;
  const int h = h0 + lane;
  const int64_t c0 = (int64_t)c * Q;
  const int len = (int)min((int64_t)Q, L - c0);
  if (h < H) {
    const float a = A[h];
    const float* d = dt + (int64_t)b * sdt + c0 * H + h;
    float s = 0.f;
#pragma unroll 8
    for (int i = 0; i < Q; ++i) {
      if (i < len) s += d[(int64_t)i * H] * a;
      sm[i * 33 + lane] = s;
    }
  }
  __syncwarp();
  const int hn = min(32, H - h0);
  for (int hl = 0; hl < hn; ++hl) {
    float* out = lam + (((int64_t)b * H + h0 + hl) * nc + c) * Q;
    for (int i = lane; i < Q; i += 32) out[i] = sm[i * 33 + hl];
  }
}

cudaError_t launch_chunk_cumsum(const Problem& p, float* lam, cudaStream_t st) {
  dim3 grid((unsigned)p.nc, (unsigned)p.B, (unsigned)ceil_div(p.H, 32));
  size_t smem = sizeof(float) * p.Q * 33;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_chunk_cumsum, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  k_chunk_cumsum<<<grid, 32, smem, st>>>(p.dt, p.sdt, p.A, lam, p.L, (int)p.H, (int)p.Q, (int)p.nc);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Step 2 (CUDA cores): chunk_states[b,h,c,n,p] = sum_s exp(lam_end - lam_s) B[s,n] x[s,p].
// grid (nc, H, B), block 256.  Thread layout: p = tid % P fixed, rows n = tid / P
// + k * (256 / P).  smem: B tile [32][N], x tile [32][P], weights [32].
// MAXE: state rows per thread, at least ceil(N / (256 / P)) (the launcher picks
// the smallest power of two), so no thread walks rows it does not own.
template <typename T, int MAXE>
__global__ void __launch_bounds__(256) k_chunk_state_simt(Problem p, const float* __restrict__ lam,
                                                          float* __restrict__ states) {
  extern __shared__ float sm[];
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int N = (int)p.N, P = (int)p.P, Q = (int)p.Q, H = (int)p.H, G = (int)p.G;
  const int g = h / (H / G);
  const int64_t c0 = (int64_t)c * Q;
  const int len = (int)min((int64_t)Q, p.L - c0);
  float* Bs = sm;
  float* xs = Bs + 32 * N;
  float* ws = xs + 32 * P;
  const float* lamc = lam + (((int64_t)b * H + h) * p.nc + c) * Q;
  const float lam_end = lamc[Q - 1];
  const T* xg = (const T*)p.x + b * p.sx + c0 * H * P + (int64_t)h * P;
  const T* Bg = (const T*)p.Bm + b * p.sbc + c0 * G * N + (int64_t)g * N;
  const int rpp = 256 / P;  // rows of the state handled per pass
  const int tid = threadIdx.x;
  const bool active = tid < rpp * P;
  const int pc = tid % P, n0 = tid / P;
  float acc[MAXE];
#pragma unroll
  for (int k = 0; k < MAXE; ++k) acc[k] = 0.f;
  for (int s0 = 0; s0 < len; s0 += 32) {
    const int sl = min(32, len - s0);
    for (int i = tid; i < 32 * N; i += 256) {
      const int j = i / N, n = i % N;
      Bs[i] = j < sl ? to_f32(Bg[(int64_t)(s0 + j) * G * N + n]) : 0.f;
    }
    for (int i = tid; i < 32 * P; i += 256) {
      const int j = i / P, q = i % P;
      xs[i] = j < sl ? to_f32(xg[(int64_t)(s0 + j) * H * P + q]) : 0.f;
    }
    if (tid < 32) ws[tid] = tid < sl ? expf(lam_end - lamc[s0 + tid]) : 0.f;
    __syncthreads();
    if (active) {
      for (int j = 0; j < sl; ++j) {
        const float wx = ws[j] * xs[j * P + pc];
        const float* brow = Bs + j * N;
#pragma unroll
        for (int k = 0; k < MAXE; ++k) {
          const int n = n0 + k * rpp;
          if (n < N) acc[k] = fmaf(wx, brow[n], acc[k]);
        }
      }
    }
    __syncthreads();
  }
  if (active) {
    float* out = states + (((int64_t)b * H + h) * p.nc + c) * N * P;
#pragma unroll
    for (int k = 0; k < MAXE; ++k) {
      const int n = n0 + k * rpp;
      if (n < N) out[(int64_t)n * P + pc] = acc[k];
    }
  }
}

cudaError_t launch_chunk_state_simt(const Problem& p, const float* lam, float* states, cudaStream_t st) {
  dim3 grid((unsigned)p.nc, (unsigned)p.H, (unsigned)p.B);
  size_t smem = sizeof(float) * (32 * p.N + 32 * p.P + 32);
  const int64_t rows = ceil_div(p.N, (int64_t)(256 / p.P));  // state rows per thread
  auto go = [&](auto tag) {
    constexpr int E = decltype(tag)::value;
    if (p.io == SSD_BF16)
      k_chunk_state_simt<__nv_bfloat16, E><<<grid, 256, smem, st>>>(p, lam, states);
    else
      k_chunk_state_simt<float, E><<<grid, 256, smem, st>>>(p, lam, states);
  };
  if (rows <= 1) go(std::integral_constant<int, 1>());
  else if (rows <= 2) go(std::integral_constant<int, 2>());
  else if (rows <= 4) go(std::integral_constant<int, 4>());
  else if (rows <= 8) go(std::integral_constant<int, 8>());
  else if (rows <= 16) go(std::integral_constant<int, 16>());
  else go(std::integral_constant<int, 32>());
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Step 3: b(c) = chunk_states(c) + exp(lam_end(c)) b(c-1), sequential over chunks,
// parallel over (b, h, n, p).  Each thread carries 4 consecutive state
// elements; lane i of a warp loads the decay of chunk cb+i and the loop
// broadcasts it with a warp shuffle.  The next chunk's input is loaded before
// the current chunk's prev state is stored (prev may alias chunk_states).
// grid (ceil(NP/512), H, B), block 128.
template <bool VEC>
__global__ void __launch_bounds__(128) k_state_passing(const float* states, const float* __restrict__ lam,
                                                       const float* init, float* prev, float* final_state,
                                                       int H, int nc, int Q, int NP) {
  grid_dep_wait();    // the chunk states and decays of the kernel before (a programmatic launch)
  grid_dep_launch();  // and the scan after it may start its prologue
  const int h = blockIdx.y, b = blockIdx.z;
  const int e0 = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  const int lane = threadIdx.x & 31;
  const bool on = e0 < NP;
  const int64_t bh = (int64_t)b * H + h;
  const float* lamb = lam + bh * nc * Q;
  const float* sin = states + bh * nc * NP + e0;
  float* pout = prev + bh * nc * NP + e0;
  float s[4] = {0.f, 0.f, 0.f, 0.f};
  auto load4 = [&](const float* ptr, float* v) {
    if (VEC) {
      const float4 t = *reinterpret_cast<const float4*>(ptr);
      v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = (e0 + i < NP) ? ptr[i] : 0.f;
    }
  };
  auto store4 = [&](float* ptr, const float* v) {
    if (VEC) {
      *reinterpret_cast<float4*>(ptr) = make_float4(v[0], v[1], v[2], v[3]);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (e0 + i < NP) ptr[i] = v[i];
    }
  };
  if (on && init) load4(init + bh * NP + e0, s);
  float nxt[4] = {0.f, 0.f, 0.f, 0.f};
  if (on) load4(sin, nxt);
  for (int cb = 0; cb < nc; cb += 32) {
    const float dec = (cb + lane < nc) ? expf(lamb[(int64_t)(cb + lane) * Q + Q - 1]) : 0.f;
    const int cn = min(32, nc - cb);
    for (int i = 0; i < cn; ++i) {
      const float d = __shfl_sync(0xffffffffu, dec, i);
      const int c = cb + i;
      float cur[4] = {nxt[0], nxt[1], nxt[2], nxt[3]};
      if (on && c + 1 < nc) load4(sin + (int64_t)(c + 1) * NP, nxt);
      if (on) store4(pout + (int64_t)c * NP, s);
#pragma unroll
      for (int k = 0; k < 4; ++k) s[k] = fmaf(d, s[k], cur[k]);
    }
  }
  if (on && final_state) store4(final_state + bh * NP + e0, s);
}

cudaError_t launch_state_passing(const Problem& p, const float* states, const float* lam, const float* init,
                                 float* prev, float* final_state, cudaStream_t st, bool programmatic) {
  const int NP = (int)(p.N * p.P);
  dim3 grid((unsigned)ceil_div(NP, 512), (unsigned)p.H, (unsigned)p.B);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = programmatic ? 1 : 0;
  const int H = (int)p.H, nc = (int)p.nc, Q = (int)p.Q;
  if (NP % 4 == 0)
    return cudaLaunchKernelEx(&cfg, k_state_passing<true>, states, lam, init, prev, final_state, H, nc, Q, NP);
  return cudaLaunchKernelEx(&cfg, k_state_passing<false>, states, lam, init, prev, final_state, H, nc, Q, NP);
}

// ---------------------------------------------------------------------------
// Step 4 (CUDA cores): y_t = sum_{s<=t} (C_t.B_s) exp(lam_t - lam_s) x_s
//                          + exp(lam_t) C_t^T prev(c) + D x_t.
// grid (nc * ceil(Q/64), H, B), block 256 = 64 rows x 4 column groups; each
// thread owns columns p = pg, pg+4, ... of one row.  smem: C rows [64][N+1],
// B tile [64][N+1], x tile [64][P+1], lam of rows and keys.
// MAXP: output columns per thread, at least ceil(P / 4) (the launcher picks the
// smallest power of two).
template <typename T, int MAXP>
__global__ void __launch_bounds__(256) k_chunk_scan_simt(Problem p, const float* __restrict__ lam,
                                                         const float* __restrict__ prev) {
  extern __shared__ float sm[];
  const int Q = (int)p.Q, N = (int)p.N, P = (int)p.P, H = (int)p.H, G = (int)p.G;
  const int ntt = (Q + 63) / 64;
  const int c = blockIdx.x / ntt, tt = blockIdx.x % ntt;
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h / (H / G);
  const int64_t c0 = (int64_t)c * Q;
  const int len = (int)min((int64_t)Q, p.L - c0);
  const int r0 = tt * 64;
  if (r0 >= len) return;  // uniform for the block
  const int nrows = min(64, len - r0);
  const int NS = N + 1, PS = P + 1;
  float* Cs = sm;
  float* Bs = Cs + 64 * NS;
  float* xs = Bs + 64 * NS;
  float* lt = xs + 64 * PS;
  float* ls = lt + 64;
  const int tid = threadIdx.x, row = tid >> 2, pg = tid & 3;
  const float* lamc = lam + (((int64_t)b * H + h) * p.nc + c) * Q;
  const T* Cg = (const T*)p.Cm + b * p.sbc + (c0 + r0) * G * N + (int64_t)g * N;
  const T* Bg = (const T*)p.Bm + b * p.sbc + c0 * G * N + (int64_t)g * N;
  const T* xg = (const T*)p.x + b * p.sx + c0 * H * P + (int64_t)h * P;
  for (int i = tid; i < 64 * N; i += 256) {
    const int j = i / N, n = i % N;
    Cs[j * NS + n] = j < nrows ? to_f32(Cg[(int64_t)j * G * N + n]) : 0.f;
  }
  if (tid < 64) lt[tid] = tid < nrows ? lamc[r0 + tid] : 0.f;
  float acc[MAXP];
#pragma unroll
  for (int k = 0; k < MAXP; ++k) acc[k] = 0.f;
  const int t = r0 + row;
  const bool active = row < nrows;
  for (int s0 = 0; s0 <= r0; s0 += 64) {
    __syncthreads();
    const int ns = min(64, len - s0);
    for (int i = tid; i < 64 * N; i += 256) {
      const int j = i / N, n = i % N;
      Bs[j * NS + n] = j < ns ? to_f32(Bg[(int64_t)(s0 + j) * G * N + n]) : 0.f;
    }
    for (int i = tid; i < 64 * P; i += 256) {
      const int j = i / P, q = i % P;
      xs[j * PS + q] = j < ns ? to_f32(xg[(int64_t)(s0 + j) * H * P + q]) : 0.f;
    }
    if (tid < 64) ls[tid] = tid < ns ? lamc[s0 + tid] : 0.f;
    __syncthreads();
    if (active) {
      const float lrow = lt[row];
      const float* crow = Cs + row * NS;
      const int jmax = min(ns - 1, t - s0);
      for (int j = 0; j <= jmax; ++j) {
        const float* brow = Bs + j * NS;
        float dot = 0.f;
        for (int n = 0; n < N; ++n) dot = fmaf(crow[n], brow[n], dot);
        const float w = dot * expf(lrow - ls[j]);
        const float* xrow = xs + j * PS;
#pragma unroll
        for (int k = 0; k < MAXP; ++k) {
          const int q = pg + 4 * k;
          if (q < P) acc[k] = fmaf(w, xrow[q], acc[k]);
        }
      }
    }
  }
  if (active) {
    const float* pv = prev + (((int64_t)b * H + h) * p.nc + c) * N * P;
    const float e = expf(lt[row]);
    const float* crow = Cs + row * NS;
    float inter[MAXP];
#pragma unroll
    for (int k = 0; k < MAXP; ++k) inter[k] = 0.f;
    for (int n = 0; n < N; ++n) {
      const float cn = crow[n];
#pragma unroll
      for (int k = 0; k < MAXP; ++k) {
        const int q = pg + 4 * k;
        if (q < P) inter[k] = fmaf(cn, pv[(int64_t)n * P + q], inter[k]);
      }
    }
    const float d = p.D ? p.D[h] : 0.f;
    const T* xt = xg + (int64_t)t * H * P;
    T* yt = (T*)p.y + b * p.sy + (c0 + t) * H * P + (int64_t)h * P;
#pragma unroll
    for (int k = 0; k < MAXP; ++k) {
      const int q = pg + 4 * k;
      if (q < P) yt[q] = from_f32<T>(acc[k] + e * inter[k] + d * to_f32(xt[q]));
    }
  }
}

cudaError_t launch_chunk_scan_simt(const Problem& p, const float* lam, const float* prev, cudaStream_t st) {
  const int64_t ntt = ceil_div(p.Q, 64);
  dim3 grid((unsigned)(p.nc * ntt), (unsigned)p.H, (unsigned)p.B);
  size_t smem = sizeof(float) * (2 * 64 * (p.N + 1) + 64 * (p.P + 1) + 128);
  const int64_t cols = ceil_div(p.P, (int64_t)4);  // output columns per thread
  cudaError_t e = cudaSuccess;
  auto go = [&](auto tag) {
    constexpr int M = decltype(tag)::value;
    if (p.io == SSD_BF16) {
      e = cudaFuncSetAttribute(k_chunk_scan_simt<__nv_bfloat16, M>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
      if (e == cudaSuccess) k_chunk_scan_simt<__nv_bfloat16, M><<<grid, 256, smem, st>>>(p, lam, prev);
    } else {
      e = cudaFuncSetAttribute(k_chunk_scan_simt<float, M>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
      if (e == cudaSuccess) k_chunk_scan_simt<float, M><<<grid, 256, smem, st>>>(p, lam, prev);
    }
  };
  if (cols <= 1) go(std::integral_constant<int, 1>());
  else if (cols <= 2) go(std::integral_constant<int, 2>());
  else if (cols <= 4) go(std::integral_constant<int, 4>());
  else if (cols <= 8) go(std::integral_constant<int, 8>());
  else go(std::integral_constant<int, 16>());
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// RMS normalisation of each row of `features` values, fp32 arithmetic,
// deterministic warp reduction.  One warp per row, eight rows per block (a
// block per row left most of its threads idle and made the launch thousands
// of tiny blocks long); with bf16 rows of a multiple of 8 values, 16-byte
// loads and stores.  in and out may alias: a lane reads each of its values
// before it writes it.
template <typename T>
__global__ void __launch_bounds__(256) k_rmsnorm(const T* in, float eps, T* out, int64_t rows, int64_t F) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= rows) return;
  const T* v = in + r * F;
  T* o = out + r * F;
  const bool vec = sizeof(T) == 2 && (F & 7) == 0 && ((reinterpret_cast<uintptr_t>(in) | reinterpret_cast<uintptr_t>(out)) & 15) == 0;
  float ss = 0.f;
  if (vec) {
    const uint4* v4 = reinterpret_cast<const uint4*>(v);
    for (int64_t f = lane; f < F / 8; f += 32) {
      const uint4 q = v4[f];
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float a = __uint_as_float(w[i] << 16), c = __uint_as_float(w[i] & 0xFFFF0000u);
        ss = fmaf(a, a, ss);
        ss = fmaf(c, c, ss);
      }
    }
  } else {
    for (int64_t f = lane; f < F; f += 32) {
      const float a = to_f32(v[f]);
      ss = fmaf(a, a, ss);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  const float inv = 1.0f / sqrtf(ss / (float)F + eps);
  if (vec) {
    const uint4* v4 = reinterpret_cast<const uint4*>(v);
    uint4* o4 = reinterpret_cast<uint4*>(o);
    for (int64_t f = lane; f < F / 8; f += 32) {
      const uint4 q = v4[f];
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
      uint32_t z[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float a = __uint_as_float(w[i] << 16) * inv, c = __uint_as_float(w[i] & 0xFFFF0000u) * inv;
        const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(a));
        const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(c));
        z[i] = lo | (hi << 16);
      }
      o4[f] = make_uint4(z[0], z[1], z[2], z[3]);
    }
  } else {
    for (int64_t f = lane; f < F; f += 32) o[f] = from_f32<T>(to_f32(v[f]) * inv);
  }
}

cudaError_t launch_rmsnorm(int64_t rows, int64_t features, int io, const void* in, float eps, void* out,
                           cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((rows + 7) / 8);
  if (io == SSD_BF16)
    k_rmsnorm<__nv_bfloat16><<<blocks, 256, 0, st>>>((const __nv_bfloat16*)in, eps, (__nv_bfloat16*)out, rows,
                                                     features);
  else
    k_rmsnorm<float><<<blocks, 256, 0, st>>>((const float*)in, eps, (float*)out, rows, features);
  return cudaGetLastError();
}

}  // namespace ssd
