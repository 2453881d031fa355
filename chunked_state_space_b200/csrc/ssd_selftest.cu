// Diagnostic kernels: one CTA computes D[128 x N] = A[128 x K] B[K x N] in
// bf16 x bf16 -> fp32 through tcgen05.mma, with the operands staged in each
// shared-memory / tensor-memory layout the scan kernels use.  A wrong
// descriptor, swizzle or TMEM packing shows up as a wrong product.
#include "ssd_selftest.h"
#include "tma.cuh"
#include "umma.cuh"

namespace ssd {

using namespace umma;

struct SelftestArgs {
  const __nv_bfloat16* A;  // variant-dependent layout, see ssd_selftest.h
  const __nv_bfloat16* B;
  float* D;                // [128][N]
  int N, K, variant;
};

__global__ void __launch_bounds__(128) k_selftest_umma(SelftestArgs a, const __grid_constant__ CUtensorMap mapA,
                                                       const __grid_constant__ CUtensorMap mapB) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar_tma, bar_mma;
  __shared__ uint32_t tmem_slot;
  const int M = 128, N = a.N, K = a.K, v = a.variant;
  const int tid = threadIdx.x, warp = tid >> 5;
  uint8_t* sA = smem;                 // 128 x K bf16 = K * 256 bytes
  uint8_t* sB = smem + K * 256;       // N x K bf16
  if (warp == 0) tmem_alloc(&tmem_slot, 256);
  if (tid == 0) {
    mbar_init(&bar_tma, 1);
    mbar_init(&bar_mma, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const bool a_mn = (v == SSD_SELFTEST_A_MN_B_MN || v == SSD_SELFTEST_A_MN_B_MN_SWAPPED);
  const bool b_mn = (v != SSD_SELFTEST_A_K_B_K);
  bool ok = true;

  if (v == SSD_SELFTEST_TMA_A_K_B_MN) {
    if (tid == 0) {
      mbar_arrive_expect_tx(&bar_tma, (uint32_t)(K * 256 + N * K * 2));
      for (int kb = 0; kb < K / 64; ++kb) tma_load_2d(sA + kb * 16384, &mapA, &bar_tma, kb * 64, 0);
      for (int nb = 0; nb < N / 64; ++nb) tma_load_2d(sB + nb * K * 128, &mapB, &bar_tma, nb * 64, 0);
    }
    ok = mbar_wait(&bar_tma, 0);
  } else {
    // manual staging with the 128-byte swizzle
    for (int i = tid; i < M * K; i += 128) {
      int m, k;
      uint32_t off;
      if (a_mn) {  // global A is [K][M]
        k = i / M; m = i % M;
        off = (m / 64) * K * 128 + swz128(k, m % 64);
      } else {     // global A is [M][K]
        m = i / K; k = i % K;
        off = (k / 64) * 16384 + swz128(m, k % 64);
      }
      *reinterpret_cast<__nv_bfloat16*>(sA + off) = a.A[i];
    }
    for (int i = tid; i < N * K; i += 128) {
      int n, k;
      uint32_t off;
      if (b_mn) {  // global B is [K][N]
        k = i / N; n = i % N;
        off = (n / 64) * K * 128 + swz128(k, n % 64);
      } else {     // global B is [N][K]
        n = i / K; k = i % K;
        off = (k / 64) * N * 128 + swz128(n, k % 64);
      }
      *reinterpret_cast<__nv_bfloat16*>(sB + off) = a.B[i];
    }
    if (v == SSD_SELFTEST_TS_A_TMEM_B_MN) {
      // row tid of A (global [M][K]) into TMEM columns N .. N + K/2, two bf16 per column
      const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)N;
      for (int c0 = 0; c0 < K / 2; c0 += 16) {
        uint32_t r[16];
        for (int j = 0; j < 16; ++j) {
          const float lo = __bfloat162float(a.A[tid * K + 2 * (c0 + j)]);
          const float hi = __bfloat162float(a.A[tid * K + 2 * (c0 + j) + 1]);
          r[j] = pack_bf16(lo, hi);
        }
        tmem_st16(lane_addr + c0, r);
      }
      tmem_wait_st();
    }
    fence_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (tid == 0 && ok) {
    const uint32_t idesc = idesc_bf16(M, N, a_mn, b_mn);
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
    for (int ks = 0; ks < K / 16; ++ks) {
      uint64_t bd;
      if (b_mn)
        bd = smem_desc(b0 + ks * 2048, K * 128, 1024);
      else
        bd = smem_desc(b0 + (ks / 4) * N * 128 + (ks % 4) * 32, 16, 1024);
      if (v == SSD_SELFTEST_TS_A_TMEM_B_MN) {
        mma_ts(tmem, tmem + (uint32_t)N + ks * 8, bd, idesc, ks > 0);
      } else {
        uint64_t ad;
        if (v == SSD_SELFTEST_A_MN_B_MN)
          ad = smem_desc(a0 + ks * 2048, K * 128, 1024);
        else if (v == SSD_SELFTEST_A_MN_B_MN_SWAPPED)
          ad = smem_desc(a0 + ks * 2048, 1024, K * 128);
        else
          ad = smem_desc(a0 + (ks / 4) * 16384 + (ks % 4) * 32, 16, 1024);
        mma_ss(tmem, ad, bd, idesc, ks > 0);
      }
    }
    mma_commit(&bar_mma);
  }
  __syncwarp();
  if (ok) ok = mbar_wait(&bar_mma, 0);
  tc_fence_after();
  if (ok) {
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    for (int c0 = 0; c0 < N; c0 += 16) {
      uint32_t r[16];
      tmem_ld16(lane_addr + c0, r);
      tmem_wait_ld();
      for (int j = 0; j < 16; ++j) a.D[tid * N + c0 + j] = __uint_as_float(r[j]);
    }
  } else if (tid == 0) {
    atomicExch(&g_device_status, 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
    tmem_relinquish();
  }
}

}  // namespace ssd

extern "C" ssd_status ssd_selftest_umma(int32_t variant, const void* A, const void* B, float* D, int32_t N,
                                        int32_t K, void* stream) {
  using namespace ssd;
  if (!A || !B || !D) return SSD_ERR_INVALID_ARG;
  if (variant < 0 || variant > SSD_SELFTEST_TMA_A_K_B_MN) return SSD_ERR_INVALID_ARG;
  if (!(N == 64 || N == 128) || !(K == 64 || K == 128 || K == 256)) return SSD_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(B) | reinterpret_cast<uintptr_t>(D)) & 15)
    return SSD_ERR_ALIGN;
  CUtensorMap mapA, mapB;
  memset(&mapA, 0, sizeof(mapA));
  memset(&mapB, 0, sizeof(mapB));
  if (variant == SSD_SELFTEST_TMA_A_K_B_MN) {
    // A [128][K] row-major: dims {K, 128}, box {64, 128}; B [K][N]: dims {N, K}, box {64, K}
    const uint64_t dA[2] = {(uint64_t)K, 128}, sA[1] = {(uint64_t)K * 2};
    const uint32_t bA[2] = {64, 128};
    const uint64_t dB[2] = {(uint64_t)N, (uint64_t)K}, sB[1] = {(uint64_t)N * 2};
    const uint32_t bB[2] = {64, (uint32_t)K};
    if (!tma::encode_bf16(&mapA, A, 2, dA, sA, bA) || !tma::encode_bf16(&mapB, B, 2, dB, sB, bB))
      return SSD_ERR_CUDA;
  }
  SelftestArgs a{static_cast<const __nv_bfloat16*>(A), static_cast<const __nv_bfloat16*>(B), D, N, K, variant};
  const size_t smem = 1024 + (size_t)K * 256 + (size_t)N * K * 2;
  cudaError_t e = cudaFuncSetAttribute(k_selftest_umma, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) {
    k_selftest_umma<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(a, mapA, mapB);
    e = cudaGetLastError();
  }
  return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

// Diagnostics for the fused kernel: the same launch as ssd_scan_fwd, with CTA
// 0 recording the clock of every pipeline event of every sub-chunk.
extern "C" ssd_status ssd_selftest_fused_trace(const ssd_dims* d, const void* x, const float* dt, const float* A,
                                               const void* Bm, const void* Cm, const float* D,
                                               const float* init_state, void* y, float* final_state,
                                               unsigned long long* trace, int64_t trace_len, void* stream) {
  using namespace ssd;
  ssd_status s = validate_dims(d);
  if (s != SSD_OK) return s;
  s = validate_scan_args(d, x, dt, A, Bm, Cm, D, init_state, y, final_state);
  if (s != SSD_OK) return s;
  Problem p = make_problem(d);
  if (!fused_supported(p)) return SSD_ERR_UNSUPPORTED;
  const int64_t ctas = p.B * p.H;
  if (!trace || trace_len < ceil_div(p.L, 128) * fused::kTraceEvents + 3 * ctas) return SSD_ERR_INVALID_ARG;
  p.x = x; p.dt = dt; p.A = A; p.Bm = Bm; p.Cm = Cm; p.D = D; p.y = y;
  return cuda_status(launch_fused_traced(p, init_state, final_state, trace, static_cast<cudaStream_t>(stream)));
}

// Timeout path of the fused kernel: the same launch as ssd_scan_fwd with its
// TMA loads withheld, so every wait on them runs out (after about a second)
// and the kernel records SSD_ERR_TIMEOUT in the device status word and
// returns; nothing faults and the context stays usable.
extern "C" ssd_status ssd_selftest_timeout(const ssd_dims* d, const void* x, const float* dt, const float* A,
                                           const void* Bm, const void* Cm, const float* D, const float* init_state,
                                           void* y, float* final_state, void* stream) {
  using namespace ssd;
  ssd_status s = validate_dims(d);
  if (s != SSD_OK) return s;
  s = validate_scan_args(d, x, dt, A, Bm, Cm, D, init_state, y, final_state);
  if (s != SSD_OK) return s;
  Problem p = make_problem(d);
  if (!fused_supported(p)) return SSD_ERR_UNSUPPORTED;
  p.x = x; p.dt = dt; p.A = A; p.Bm = Bm; p.Cm = Cm; p.D = D; p.y = y;
  return cuda_status(launch_fused_withheld(p, init_state, final_state, static_cast<cudaStream_t>(stream)));
}

// Carry path of the two-head kernel: the segmented schedule of ssd_scan_fwd with
// no carry ever published, so every segment after the first waits for its
// predecessor's state until its bounded wait runs out (about two seconds),
// records SSD_ERR_TIMEOUT and drains; nothing faults.
extern "C" ssd_status ssd_selftest_carry_timeout(const ssd_dims* d, const void* x, const float* dt, const float* A,
                                                 const void* Bm, const void* Cm, const float* D,
                                                 const float* init_state, void* y, float* final_state,
                                                 void* workspace, size_t workspace_bytes, void* stream) {
  using namespace ssd;
  ssd_status s = validate_dims(d);
  if (s != SSD_OK) return s;
  s = validate_scan_args(d, x, dt, A, Bm, Cm, D, init_state, y, final_state);
  if (s != SSD_OK) return s;
  Problem p = make_problem(d);
  if (!uses_pair_kernel(p) || pair_workspace_bytes(p) == 0) return SSD_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < pair_workspace_bytes(p)) return SSD_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0) return SSD_ERR_ALIGN;
  p.x = x; p.dt = dt; p.A = A; p.Bm = Bm; p.Cm = Cm; p.D = D; p.y = y;
  return cuda_status(
      launch_pair(p, init_state, final_state, workspace, workspace_bytes, static_cast<cudaStream_t>(stream), 2));
}

// Segments per sequence of the two-head kernel's schedule for the following
// launches of this process (0 restores the choice from the shape).
extern "C" ssd_status ssd_selftest_set_segments(int nseg) {
  if (nseg < 0) return SSD_ERR_INVALID_ARG;
  ssd::set_pair_segments(nseg);
  ssd::set_fused_segments(nseg);
  return SSD_OK;
}

// Chunks per CTA of the tensor-core step kernels for the following launches.
extern "C" ssd_status ssd_selftest_set_step_chunks(int n) {
  if (n < 0) return SSD_ERR_INVALID_ARG;
  ssd::set_step_chunks_per_cta(n);
  return SSD_OK;
}

// The one-head kernel's segmented form for the following launches: the first
// `whole` sequences whole, every later one in about nseg segments.
extern "C" ssd_status ssd_selftest_set_split(int nseg, int64_t whole) {
  if (nseg < 0 || whole < 0) return SSD_ERR_INVALID_ARG;
  ssd::set_fused_split(nseg, whole);
  return SSD_OK;
}
