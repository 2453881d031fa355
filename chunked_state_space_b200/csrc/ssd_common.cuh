// Internal definitions shared by the CUDA sources of libssd (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ssd.h"

namespace ssd {

// One layer of the scan as the kernels see it.  Batch strides (in elements)
// let the vertical schedule run the kernels on V-token slices of full-length
// tensors without copies; every other dimension is contiguous.
struct Problem {
  int64_t B, L, H, P, N, G, Q, nc;
  int io;  // SSD_F32 / SSD_BF16
  const void* x;
  int64_t sx;  // batch stride of x (default L*H*P)
  const float* dt;
  int64_t sdt;  // batch stride of dt (default L*H)
  const float* A;
  const void* Bm;
  const void* Cm;
  int64_t sbc;  // batch stride of Bm and Cm (default L*G*N)
  const float* D;
  void* y;
  int64_t sy;  // batch stride of y (default L*H*P)
  // token strides (elements); the contiguous layout has ldx = ldy = H*P,
  // lddt = H, ldbc = G*N.  Only the fused tensor-core kernel reads them.
  int64_t ldx, lddt, ldbc, ldy;
  int input_dt;     // SSD_FLAG_INPUT_DT: the input term is dt_t B_t x_t^T
  int two_heads;    // SSD_FLAG_TWO_HEADS_PER_CTA: the two-head kernel where it applies
};

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Device status word raised by bounded waits that gave up (read and cleared
// by ssd_read_device_status).  libssd is one translation unit, so this is its
// only definition.
__device__ int g_device_status = 0;

// Programmatic dependent launch: a kernel launched with the programmatic
// stream-serialization attribute may start while the kernel before it on the
// stream still runs; grid_dep_wait() returns once that kernel has completed
// and its memory is visible (at once for an ordinary launch), and
// grid_dep_launch() lets the next such kernel start early.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launchers of the CUDA-core kernels (ssd_simt.cu).  They return
// cudaSuccess or the launch error.
cudaError_t launch_chunk_cumsum(const Problem& p, float* lam, cudaStream_t st);
cudaError_t launch_chunk_state_simt(const Problem& p, const float* lam, float* states, cudaStream_t st);
// programmatic: launched so that it may start while the kernel before it on
// the stream finishes (it waits for that kernel's results itself)
cudaError_t launch_state_passing(const Problem& p, const float* states, const float* lam,
                                 const float* init, float* prev, float* final_state, cudaStream_t st,
                                 bool programmatic = false);
cudaError_t launch_chunk_scan_simt(const Problem& p, const float* lam, const float* prev, cudaStream_t st);
cudaError_t launch_ssd_step(const Problem& p, float* state, cudaStream_t st);
cudaError_t launch_rmsnorm(int64_t rows, int64_t features, int io, const void* in, float eps, void* out,
                           cudaStream_t st);

}  // namespace ssd
