// End states of sequence segments from a zero start, for the segmented form
// of the one-head scan (the page's chunk decomposition one level up,
// "分块推理：解锁循环模型并行计算，实现长序列高效处理" §2.1-§2.2, with a segment as the chunk).
//
// Unrolled over a segment of tokens s = 0 .. S-1 the recurrence gives its end
// state from a zero start as one sum,
//   h_end = sum_s exp(A_h (tau_end - tau_s)) B_s x_s^T,
// tau the running sum of dt, so tau_end - tau_s is the dt of the tokens after
// s.  Folding that decay into the rows of x (X''_s = w_s x_s, w_s <= 1; with
// the dt-scaled input w_s also carries dt_s) leaves a plain product
// h_end = B^T X'' over the whole segment: the tensor core accumulates every
// 128-token tile into one TMEM accumulator, with no state update between
// tiles.  The tiles are walked from the segment's end backwards, so each
// token's suffix sum of dt is accumulated directly (sums of non-negative
// terms, no differences of large running sums).  The segment's total
// log-decay A_h tau_end comes out of the same walk.
//
// One CTA per segment: warp 0 issues the TMA loads (x and B tiles, four
// stages, with an L2 prefetch eight tiles ahead), warp 1 owns the 64 TMEM columns and issues the MMAs, warps 2-5
// scan dt and scale the x rows in place, and at the end read the accumulator
// out (warp w reads TMEM lane quarter w % 4).  The kernel streams x from HBM;
// every wait is bounded and a timeout raises the device status word.
#include <atomic>

#include "ssd_common.cuh"
#include "ssd_split.cuh"
#include "ssd_tc.cuh"
#include "tma.cuh"
#include "umma.cuh"

namespace ssd {
namespace lean {

using namespace umma;

constexpr int T = 128;       // tokens per tile
constexpr int P = 64;        // head dim
constexpr int STAGES = 4;
constexpr int THREADS = 192;
constexpr int BUILD = 128;   // threads of warps 2-5
constexpr uint32_t TILE = 16384;             // [128 rows][64 bf16], 128-byte swizzled
constexpr uint32_t STAGE = 3 * TILE;         // x, B (two 64-column halves)
constexpr uint32_t OFF_X = 0, OFF_B = TILE;
constexpr uint32_t OFF_RED = STAGES * STAGE;           // float [2][4]: per-warp dt totals (two slots)
constexpr uint32_t OFF_BAR = OFF_RED + 64;
enum { FULL0 = 0, READY0 = STAGES, EMPTY0 = 2 * STAGES, DONE = 3 * STAGES, NBAR = 3 * STAGES + 1 };
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
constexpr uint32_t TMEM_COLS = 64;
constexpr float kLog2e = 1.4426950408889634f;

struct Params {
  int64_t L, Q;          // sequence length; segment length (a multiple of 128)
  int H, G, nc;          // heads, groups, segments per sequence
  int64_t seq0, nseq;    // first sequence (batch * H + head) of the grid, and their count
  const float* dt;
  int64_t sdt, lddt;     // batch and token strides of dt
  const float* A;
  int input_dt;          // the input term is dt_t B_t x_t^T
  float* states;         // [slots][N][P] end state of each segment (slot (seq - seq0) * nc + segment)
  float* seg_decay;      // [slots] A_h * (sum of dt over the segment)
};

// Bounded mbarrier wait (1 s, %globaltimer): false on timeout, after raising
// the device status word and the CTA's abort flag.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    if ((spin & 31) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > 1000000000ull) {
        *abort = 1;
        atomicExch(&g_device_status, 2);
        return false;
      }
    }
  }
}

__device__ __forceinline__ void named_bar_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n)); }
// 2^x with the ex2.approx PTX instruction (flushes denormals; |rel err| ~ 2^-22).
__device__ __forceinline__ float ex2f_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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

__global__ void __launch_bounds__(THREADS, 1)
    k_ssd_segment_states(Params p, const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_b) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(sm);
  float* red = reinterpret_cast<float*>(sm + OFF_RED);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_MISC + 4);

  grid_dep_launch();  // the combine may be scheduled now (it waits for this grid's results)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // sequence-fastest: CTAs that run together read the same tokens of
  // neighbouring heads (whole rows of x, shared tiles of B)
  const int64_t bh = p.seq0 + (int64_t)blockIdx.x % p.nseq;
  const int seg = (int)((int64_t)blockIdx.x / p.nseq);
  const int64_t slot = (bh - p.seq0) * p.nc + seg;
  const int b = (int)(bh / p.H), h = (int)(bh % p.H);
  const int g = h / (p.H / p.G);
  const int64_t t_seg = (int64_t)seg * p.Q;                     // first token of the segment
  const int ntile = (int)ceil_div(min(p.Q, p.L - t_seg), (int64_t)T);

  if (warp == 1) tmem_alloc(tmem_slot, TMEM_COLS);
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&bar[FULL0 + i], 1);
      mbar_init(&bar[READY0 + i], BUILD);
      mbar_init(&bar[EMPTY0 + i], 1);
    }
    mbar_init(&bar[DONE], 1);
    fence_mbar_init();
    prefetch_tmap(&map_x);
    prefetch_tmap(&map_b);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // L2 prefetch runs kPrefetch tiles ahead of the shared-memory loads, so a
      // stage freed by the MMAs refills from L2 rather than from DRAM
      constexpr int kPrefetch = 8;
      auto prefetch = [&](int i) {
        if (i >= ntile) return;
        const int t0 = (int)(t_seg + (int64_t)(ntile - 1 - i) * T);
        tma_prefetch_4d(&map_x, 0, h, t0, b);
        tma_prefetch_4d(&map_b, 0, g, t0, b);
        tma_prefetch_4d(&map_b, 64, g, t0, b);
      };
      for (int i = 0; i < kPrefetch; ++i) prefetch(i);
      int issued = 0;
      for (int i = 0; i < ntile; ++i) {  // tiles from the segment's end backwards
        const int st = i % STAGES;
        prefetch(i + kPrefetch);
        if (i >= STAGES && !wait_bar(&bar[EMPTY0 + st], ((i / STAGES) + 1) & 1, abort_flag)) break;
        const int t0 = (int)(t_seg + (int64_t)(ntile - 1 - i) * T);
        uint8_t* sx = sm + st * STAGE;
        mbar_arrive_expect_tx(&bar[FULL0 + st], STAGE);
        tma_load_4d(sx + OFF_X, &map_x, &bar[FULL0 + st], 0, h, t0, b);
        tma_load_4d(sx + OFF_B, &map_b, &bar[FULL0 + st], 0, g, t0, b);
        tma_load_4d(sx + OFF_B + TILE, &map_b, &bar[FULL0 + st], 64, g, t0, b);
        issued = i + 1;
      }
      // the loads issued to each stage land before the CTA may exit
      for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&bar[FULL0 + i % STAGES], (i / STAGES) & 1) && globaltimer_ns() - t0 < 1000000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idB = idesc_bf16(128, 64, true, true);       // B^T (MN-major) x X'' (MN-major)
      const uint64_t dB = smem_desc(sbase + OFF_B, TILE, 1024);
      const uint64_t dX = smem_desc(sbase + OFF_X, TILE, 1024);
      for (int i = 0; i < ntile; ++i) {
        const int st = i % STAGES;
        if (!wait_bar(&bar[READY0 + st], (i / STAGES) & 1, abort_flag)) break;
        tc_fence_after();
        const uint64_t cB = desc_advance(dB, st * STAGE), cX = desc_advance(dX, st * STAGE);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)  // h_end += B^T X'' over the tile's 128 tokens
          mma_ss(tmem, desc_advance(cB, ks * 2048), desc_advance(cX, ks * 2048), idB, (i > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&bar[EMPTY0 + st]);
      }
      // every MMA issued completes before the accumulator is read (also on abort)
      mma_commit(&bar[DONE]);
    }
  } else {
    // ------------------------------------------------------------ dt scan, X'', read-out
    const int r = threadIdx.x - 64;   // token row of the tile
    const int wb = r >> 5;            // builder warp 0..3
    const float Al = p.A[h] * kLog2e;
    const float* dtb = p.dt + (int64_t)b * p.sdt + h;
    auto load_dt = [&](int i) {
      const int64_t t = t_seg + (int64_t)(ntile - 1 - i) * T + r;
      return (i < ntile && t < p.L) ? dtb[t * p.lddt] : 0.f;
    };
    float tau_after = 0.f;  // sum of dt over the tiles already walked (the later tokens)
    // dt of the next three tiles in flight (a token's dt is a scattered 4-byte load)
    float dq0 = load_dt(0), dq1 = load_dt(1), dq2 = load_dt(2);
    bool ok = true;
    for (int i = 0; i < ntile; ++i) {
      const int st = i % STAGES;
      const float d = dq0;
      dq0 = dq1;
      dq1 = dq2;
      dq2 = load_dt(i + 3);
      // suffix sums over the tile: incl = dt of tokens r .. 127, excl = of r+1 .. 127
      float incl = d;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float v = __shfl_down_sync(0xffffffffu, incl, off);
        if (lane + off < 32) incl += v;
      }
      float* rs = red + (i & 1) * 4;  // two slots: a warp may run a tile ahead of the others
      if (lane == 0) rs[wb] = incl;
      named_bar_sync(1, BUILD);
      float later = 0.f;  // dt of the tiles' warps after this one
      for (int k = wb + 1; k < 4; ++k) later += rs[k];
      const float total = rs[0] + rs[1] + rs[2] + rs[3];
      float excl = __shfl_down_sync(0xffffffffu, incl, 1);
      if (lane == 31) excl = 0.f;
      excl += later;
      float w = ex2f_approx((excl + tau_after) * Al);
      if (p.input_dt) w *= d;
      tau_after += total;
      // X''_r = w x_r in place (fp32 product, one bf16 rounding)
      if (ok) ok = wait_bar(&bar[FULL0 + st], (i / STAGES) & 1, abort_flag);
      if (ok) {
        const uint32_t row = sbase + st * STAGE + OFF_X;
        const float2 w2 = make_float2(w, w);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t a = row + swz128((uint32_t)r, (uint32_t)(8 * c));
          uint4 v;
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                       : "r"(a));
          uint32_t* u = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f = mul2(make_float2(__uint_as_float(u[k] << 16), __uint_as_float(u[k] & 0xFFFF0000u)), w2);
            u[k] = pack_bf16(f.x, f.y);
          }
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                       : "memory");
        }
        fence_async_smem();  // X'' is read by the MMA (async proxy)
      }
      mbar_arrive(&bar[READY0 + st]);
    }
    // the accumulator: state row n = this warp's lane quarter * 32 + lane
    const bool done = wait_bar(&bar[DONE], 0, abort_flag);
    tc_fence_after();
    const int q = warp & 3;
    const int n = q * 32 + lane;
    float* dst = p.states + slot * (int64_t)(128 * P) + (int64_t)n * P;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint32_t v[32];
      tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + 32 * c, v);
      tmem_wait_ld();
      if (done) {
#pragma unroll
        for (int k = 0; k < 32; k += 4)
          *reinterpret_cast<float4*>(dst + 32 * c + k) =
              make_float4(__uint_as_float(v[k]), __uint_as_float(v[k + 1]), __uint_as_float(v[k + 2]),
                          __uint_as_float(v[k + 3]));
      }
    }
    if (r == 0 && p.seg_decay) p.seg_decay[slot] = p.A[h] * tau_after;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
    tmem_relinquish();
  }
}


// Step 2 of the step-by-step scan on tensor cores: the end state of every
// chunk from a zero start, states[b,h,c] = sum over the chunk's tokens s of
// exp(lam_end(c) - lam(c, s)) B_s x_s^T, with lam the chunk-local cumulative
// sums of dt * A from step 1.  The same product as above, accumulated over
// the chunk's tiles; one CTA walks cpb consecutive chunks of one (batch, head)
// so its TMA pipeline stays full across chunk boundaries, and the read-out of
// chunk c (two TMEM accumulators, 128 columns) overlaps the MMAs of chunk c+1.
struct ChunkParams {
  int64_t L, Q, nc;   // sequence length, chunk length (a multiple of 128), chunks per sequence
  int H, G, cpb;      // heads, groups, chunks per CTA
  int64_t nseq;       // B * H
  const float* lam;   // [B,H,nc,Q] chunk-local cumulative sums of dt * A
  float* states;      // [B,H,nc,N,P]
};

enum { CFULL0 = 3 * STAGES, CFREE0 = 3 * STAGES + 2, NBAR_C = 3 * STAGES + 4 };
constexpr uint32_t SMEM_BYTES_C = OFF_BAR + NBAR_C * 8 + 16 + 1024;  // + alignment slack

__global__ void __launch_bounds__(THREADS, 1)
    k_ssd_chunk_states(ChunkParams p, const __grid_constant__ CUtensorMap map_x,
                       const __grid_constant__ CUtensorMap map_b) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(sm);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_BAR + NBAR_C * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_BAR + NBAR_C * 8 + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // sequence-fastest, as the other chunk grids
  const int64_t bh = (int64_t)blockIdx.x % p.nseq;
  const int64_t c0 = (int64_t)blockIdx.x / p.nseq * p.cpb;          // first chunk of this CTA
  const int nch = (int)min((int64_t)p.cpb, p.nc - c0);              // chunks of this CTA
  const int b = (int)(bh / p.H), h = (int)(bh % p.H);
  const int g = h / (p.H / p.G);
  auto tiles_of = [&](int i) {  // tiles of the CTA's chunk i (the sequence's last chunk may be short)
    const int64_t t0 = (c0 + i) * p.Q;
    return (int)ceil_div(min(p.Q, p.L - t0), (int64_t)T);
  };

  if (warp == 1) tmem_alloc(tmem_slot, 2 * TMEM_COLS);
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&bar[FULL0 + i], 1);
      mbar_init(&bar[READY0 + i], BUILD);
      mbar_init(&bar[EMPTY0 + i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[CFULL0 + i], 1);
      mbar_init(&bar[CFREE0 + i], BUILD);
    }
    fence_mbar_init();
    prefetch_tmap(&map_x);
    prefetch_tmap(&map_b);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int k = 0, issued = 0;  // tile counter over the CTA's chunks
      bool ok = true;
      for (int i = 0; i < nch && ok; ++i) {
        const int nt = tiles_of(i);
        for (int tt = 0; tt < nt; ++tt, ++k) {
          const int st = k % STAGES;
          if (k >= STAGES && !wait_bar(&bar[EMPTY0 + st], ((k / STAGES) + 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const int t0 = (int)((c0 + i) * p.Q + (int64_t)tt * T);
          uint8_t* sx = sm + st * STAGE;
          mbar_arrive_expect_tx(&bar[FULL0 + st], STAGE);
          tma_load_4d(sx + OFF_X, &map_x, &bar[FULL0 + st], 0, h, t0, b);
          tma_load_4d(sx + OFF_B, &map_b, &bar[FULL0 + st], 0, g, t0, b);
          tma_load_4d(sx + OFF_B + TILE, &map_b, &bar[FULL0 + st], 64, g, t0, b);
          issued = k + 1;
        }
      }
      for (int q = (issued > STAGES ? issued - STAGES : 0); q < issued; ++q) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&bar[FULL0 + q % STAGES], (q / STAGES) & 1) && globaltimer_ns() - t0 < 1000000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idB = idesc_bf16(128, 64, true, true);
      const uint64_t dB = smem_desc(sbase + OFF_B, TILE, 1024);
      const uint64_t dX = smem_desc(sbase + OFF_X, TILE, 1024);
      int k = 0;
      bool ok = true;
      for (int i = 0; i < nch && ok; ++i) {
        const int a = i & 1;
        // the accumulator of chunk i-2 has been read out
        if (i >= 2 && !wait_bar(&bar[CFREE0 + a], ((i - 2) >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        const int nt = tiles_of(i);
        for (int tt = 0; tt < nt; ++tt, ++k) {
          const int st = k % STAGES;
          if (!wait_bar(&bar[READY0 + st], (k / STAGES) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t cB = desc_advance(dB, st * STAGE), cX = desc_advance(dX, st * STAGE);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_ss(tmem + a * TMEM_COLS, desc_advance(cB, ks * 2048), desc_advance(cX, ks * 2048), idB,
                   (tt > 0 || ks > 0) ? 1u : 0u);
          mma_commit(&bar[EMPTY0 + st]);
        }
        mma_commit(&bar[CFULL0 + a]);  // chunk i's state is complete (also after an abort)
      }
    }
  } else {
    // ------------------------------------------------------------ weights, X'', read-out
    const int r = threadIdx.x - 64;   // token row of the tile
    const int q = warp & 3;           // TMEM lane quarter of the read-out
    const int n = q * 32 + lane;      // state row n of the read-out
    const float* lamh = p.lam + bh * p.nc * p.Q;
    auto read_out = [&](int i) {      // chunk i's accumulator to states[b,h,c0+i]
      const int a = i & 1;
      const bool done = wait_bar(&bar[CFULL0 + a], (i >> 1) & 1, abort_flag);
      tc_fence_after();
      float* dst = p.states + ((bh * p.nc + c0 + i) * 128 + n) * (int64_t)P;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + a * TMEM_COLS + 32 * c, v);
        tmem_wait_ld();
        if (done) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + 32 * c + e) =
                make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]), __uint_as_float(v[e + 2]),
                            __uint_as_float(v[e + 3]));
        }
      }
      tc_fence_before();
      mbar_arrive(&bar[CFREE0 + a]);
    };
    int k = 0;
    bool ok = true;
    for (int i = 0; i < nch; ++i) {
      const float* lc = lamh + (c0 + i) * p.Q;
      const float lend = lc[p.Q - 1] * kLog2e;  // past L, lam stays at its last value
      const int nt = tiles_of(i);
      for (int tt = 0; tt < nt; ++tt, ++k) {
        const int st = k % STAGES;
        const float w = ex2f_approx(lend - lc[tt * T + r] * kLog2e);
        if (ok) ok = wait_bar(&bar[FULL0 + st], (k / STAGES) & 1, abort_flag);
        if (ok) {
          const uint32_t row = sbase + st * STAGE + OFF_X;
          const float2 w2 = make_float2(w, w);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t ad = row + swz128((uint32_t)r, (uint32_t)(8 * c));
            uint4 v;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(ad));
            uint32_t* u = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f =
                  mul2(make_float2(__uint_as_float(u[e] << 16), __uint_as_float(u[e] & 0xFFFF0000u)), w2);
              u[e] = pack_bf16(f.x, f.y);
            }
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(ad), "r"(v.x), "r"(v.y), "r"(v.z),
                         "r"(v.w)
                         : "memory");
          }
          fence_async_smem();
        }
        mbar_arrive(&bar[READY0 + st]);
      }
      if (i > 0) read_out(i - 1);  // overlaps the MMAs of chunk i
    }
    if (nch > 0) read_out(nch - 1);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * TMEM_COLS);
    tmem_relinquish();
  }
}

}  // namespace lean

// The segments of sequences seq0, seq0 + 1, ... (p.Q = the segment length, a
// multiple of 128; p.nc segments per sequence): each segment's end state from
// a zero start into states[slot] and its total log-decay into seg_decay[slot],
// slot = (sequence - seq0) * nc + segment.
cudaError_t launch_segment_states(const Problem& p, int64_t seq0, float* states, float* seg_decay, cudaStream_t st) {
  using namespace lean;
  if (!p.x || !p.Bm || !p.dt || !p.A || !states || p.Q % T != 0 || p.P != P || p.N != 128) return cudaErrorInvalidValue;
  const int64_t ctas = (p.B * p.H - seq0) * p.nc;
  if (seq0 < 0 || ctas <= 0 || ctas >= (1ll << 31)) return cudaErrorInvalidValue;
  CUtensorMap mx, mb;
  const uint32_t box[4] = {64, 1, (uint32_t)T, 1};
  const uint64_t dx[4] = {(uint64_t)P, (uint64_t)p.H, (uint64_t)p.L, (uint64_t)p.B};
  const uint64_t sx[3] = {(uint64_t)P * 2, (uint64_t)p.ldx * 2, (uint64_t)p.sx * 2};
  const uint64_t dbc[4] = {(uint64_t)128, (uint64_t)p.G, (uint64_t)p.L, (uint64_t)p.B};
  const uint64_t sbc[3] = {(uint64_t)128 * 2, (uint64_t)p.ldbc * 2, (uint64_t)p.sbc * 2};
  if (!tma::encode_bf16_4d_cached(&mx, p.x, dx, sx, box) || !tma::encode_bf16_4d_cached(&mb, p.Bm, dbc, sbc, box))
    return cudaErrorInvalidValue;
  Params kp;
  kp.L = p.L;
  kp.Q = p.Q;
  kp.H = (int)p.H;
  kp.G = (int)p.G;
  kp.nc = (int)p.nc;
  kp.seq0 = seq0;
  kp.nseq = p.B * p.H - seq0;
  kp.dt = p.dt;
  kp.sdt = p.sdt;
  kp.lddt = p.lddt;
  kp.A = p.A;
  kp.input_dt = p.input_dt;
  kp.states = states;
  kp.seg_decay = seg_decay;
  static std::atomic<unsigned long long> attr_set{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set.load() & bit)) {
    e = cudaFuncSetAttribute((const void*)k_ssd_segment_states, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit);
  }
  k_ssd_segment_states<<<(unsigned)ctas, THREADS, SMEM_BYTES, st>>>(kp, mx, mb);
  return cudaGetLastError();
}

}  // namespace ssd

namespace ssd {
static int g_step_cpc = 0;  // forced by a self-test (0: chosen from the shape)
void set_step_chunks_per_cta(int n) { g_step_cpc = n > 0 ? n : 0; }
// Consecutive chunks per CTA of the tensor-core step kernels (steps 2 and 4):
// up to 16 tiles per CTA (a CTA's pipeline fill is a few tiles' time), fewer
// where that would leave less than four CTAs per SM.
int64_t step_chunks_per_cta(const Problem& p) {
  int64_t cpc = g_step_cpc > 0 ? g_step_cpc : ceil_div((int64_t)16, p.Q / lean::T);
  if (g_step_cpc <= 0) {
    const int64_t nseq = p.B * p.H, want = 4 * (int64_t)split::sm_count();
    while (cpc > 1 && nseq * ceil_div(p.nc, cpc) < want) cpc = ceil_div(cpc, (int64_t)2);
  }
  return cpc < p.nc ? cpc : (p.nc > 0 ? p.nc : 1);
}

// Step 2 of the step-by-step scan on tensor cores (bf16, P = 64, N = 128, Q a
// multiple of 128): chunk_states[b,h,c] from a zero start, lam from step 1.
cudaError_t launch_chunk_states_seq(const Problem& p, const float* lam, float* states, cudaStream_t st) {
  using namespace lean;
  if (!p.x || !p.Bm || !lam || !states || p.Q % T != 0 || p.P != P || p.N != 128) return cudaErrorInvalidValue;
  const int64_t nseq = p.B * p.H;
  const int64_t cpb = step_chunks_per_cta(p);
  const int64_t ctas = nseq * ceil_div(p.nc, cpb);
  if (ctas <= 0 || ctas >= (1ll << 31)) return cudaErrorInvalidValue;
  CUtensorMap mx, mb;
  const uint32_t box[4] = {64, 1, (uint32_t)T, 1};
  const uint64_t dx[4] = {(uint64_t)P, (uint64_t)p.H, (uint64_t)p.L, (uint64_t)p.B};
  const uint64_t sx[3] = {(uint64_t)P * 2, (uint64_t)p.ldx * 2, (uint64_t)p.sx * 2};
  const uint64_t dbc[4] = {(uint64_t)128, (uint64_t)p.G, (uint64_t)p.L, (uint64_t)p.B};
  const uint64_t sbc[3] = {(uint64_t)128 * 2, (uint64_t)p.ldbc * 2, (uint64_t)p.sbc * 2};
  if (!tma::encode_bf16_4d_cached(&mx, p.x, dx, sx, box) || !tma::encode_bf16_4d_cached(&mb, p.Bm, dbc, sbc, box))
    return cudaErrorInvalidValue;
  ChunkParams kp;
  kp.L = p.L;
  kp.Q = p.Q;
  kp.nc = p.nc;
  kp.H = (int)p.H;
  kp.G = (int)p.G;
  kp.cpb = (int)cpb;
  kp.nseq = nseq;
  kp.lam = lam;
  kp.states = states;
  static std::atomic<unsigned long long> attr_set{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set.load() & bit)) {
    e = cudaFuncSetAttribute((const void*)k_ssd_chunk_states, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES_C);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit);
  }
  k_ssd_chunk_states<<<(unsigned)ctas, THREADS, SMEM_BYTES_C, st>>>(kp, mx, mb);
  return cudaGetLastError();
}
}  // namespace ssd
