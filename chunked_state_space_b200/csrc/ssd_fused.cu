// Fused tensor-core kernel of the chunked SSD scan (sm_100a): all four steps
// of "分块推理：解锁循环模型并行计算，实现长序列高效处理" §2.1-§2.2 in one pass, with the
// inter-chunk state carried on chip.
//
// One CTA owns one (batch, head) sequence and walks it in 128-token
// sub-chunks j (a Q = 256 chunk is two of them: the page's intra/inter split
// applied once more inside the chunk, which is exact by its §2.3).  Per
// sub-chunk, with lam the in-sub-chunk cumulative sum of dt*A:
//   S       = C_j B_j^T                                   (tcgen05, 128x128x128)
//   P       = S (.) exp(lam_t - lam_s) [s <= t]  -> bf16 in TMEM, columns 0-63
//   y_intra = P X_j                               (A operand from TMEM)
//   y_inter = C_j bf16(s_{j-1})                   (into S columns 64-127, dead by then)
//   b_intra = B_j^T X'_j,  X'_j = diag(exp(lam_end - lam_s)) X_j
//   (with the dt-scaled input every column s of P and row s of X' also
//   carries dt_s)
//   y_t     = y_intra + exp(lam_t) y_inter + D x_t    (fp32; x_j copied from its stage
//             tile into TMEM, over P's first 32 columns once the products are done)
//   s_j     = exp(lam_end) s_{j-1} + b_intra              (fp32, registers)
// Warp roles (384 threads): warp 2 issues TMA loads; warp 3 owns TMEM and
// issues MMAs; warps 0-1 load dt one sub-chunk ahead, scan lam, form the
// per-column decay factors and X'; warps 4-7 (one thread per row) turn S
// into P; warps 8-11 (one thread per row) finish y, update the state and
// publish its bf16 copy.  The mask needs exp(lam_t - lam_s) only inside the
// diagonal 32x32 blocks: below them it is exp(lam_t - lam_r) exp(lam_r - lam_s)
// with r the last column of the block (both factors <= 1).
// TMEM holds two 256-column buffers [S -> P -> x | y_inter][y_intra][b_intra] so sub-chunk
// j+1's S and mask overlap sub-chunk j's products and epilogue.  Every wait is bounded; a timeout
// raises g_device_status and the roles drain without further waits.
#include <atomic>

#include "ssd_split.cuh"
#include "ssd_tc.cuh"
#include "tma.cuh"
#include "umma.cuh"

namespace ssd {
namespace fused {

using namespace umma;

constexpr int T = 128;       // tokens per sub-chunk
constexpr int P = 64;        // head dim
constexpr int NS = 128;      // state dim
constexpr int THREADS = 384;
constexpr uint32_t TILE = 16384;               // [128 rows][64 bf16], 128B-swizzled
constexpr uint32_t STAGE = 5 * TILE;           // X, B (2 blocks), C (2 blocks)
constexpr uint32_t OFF_X = 0, OFF_B = TILE, OFF_C = 3 * TILE;
constexpr uint32_t OFF_XP = 2 * STAGE;         // X' (two buffers)
constexpr uint32_t OFF_PREV = OFF_XP + 2 * TILE;  // bf16 state, MN-major [n][p]
constexpr uint32_t OFF_LAM = OFF_PREV + TILE;  // float [4][128]
constexpr uint32_t OFF_ECOL = OFF_LAM + 4 * T * 4;  // float [4][128]
constexpr uint32_t OFF_DTS = OFF_ECOL + 4 * T * 4;   // float [4][128]: the input term's column factor
                                                     // (dt_s, times r_s with the normalised input)
constexpr uint32_t OFF_RN = OFF_DTS + 4 * T * 4;     // float [4][128]: r_t of the normalised input
constexpr uint32_t OFF_WTOT = OFF_RN + 4 * T * 4;
constexpr uint32_t OFF_BAR = OFF_WTOT + 64;
constexpr uint32_t NBAR = 22;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 64 + 1024;  // + alignment slack
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TX_BYTES = 5 * TILE;

// Modes: the whole scan (one CTA per (batch, head) sequence), or one CTA per
// (batch, head, chunk) for the step kernels -- chunk states from a zero start
// (step 2) or chunk outputs from given previous states (step 4) -- with the
// log-decay sums read from step 1's output instead of scanned from dt.
enum { MODE_SCAN = 0, MODE_CHUNK_STATE = 1, MODE_CHUNK_SCAN = 2 };

struct Params {
  int mode;
  int64_t L;
  int H, G, nsub;
  int64_t nc, Q;         // chunking of the step kernels
  const float* lam_in;   // step-1 log-decay sums [B,H,nc,Q] (step modes), or NULL: the
                         // kernel scans dt itself from the chunk's first token
  const float* dt;
  int64_t sdt, lddt;  // batch and token strides of dt
  int input_dt;       // the input term is dt_t B_t x_t^T
  const float* A;
  const float* D;
  const float* init;         // whole-sequence CTAs: [B*H][N][P] initial states, or NULL
  float* final_state;        // whole-sequence CTAs: [B*H][N][P] final states, or NULL
  const float* chunk_init;   // chunk-scan CTAs: [slots][N][P] start state of each chunk
  float* chunk_final;        // chunk-state CTAs: [slots][N][P] end state of each chunk
  // Grid layout: the first `whole` CTAs scan sequences 0..whole-1 whole (step
  // modes with whole > 0 are mixed grids); the rest run the step mode over
  // the nseq sequences seq0, seq0+1, ..., one CTA per chunk, sequence-fastest
  // (CTAs that run together read the same tokens of neighbouring heads: whole
  // rows of x, shared tiles of B and C), chunk slot (sequence - seq0) * nc +
  // chunk.
  int64_t whole, seq0, nseq;
  int cpc;  // MULTI: chunks per CTA (consecutive chunks of one sequence; state reloaded at each)
  const __nv_bfloat16* x;
  int64_t sx, ldx;    // batch and token strides of x
  __nv_bfloat16* y;
  int64_t sy;
  // RMS-normalised input (layer stacks): the input rows are the previous
  // layer's stored y, and each token t enters as r_t x_t with
  // r_t = 1 / sqrt(sum over heads of ss_in[b, t, h] / (H P) + eps)
  const float* ss_in;   // [B][L][H] sums of squares of the input rows per (token, head), or NULL
  float* ss_out;        // [B][L][H] sums of squares of this call's stored (bf16) y rows, or NULL
  int64_t sss;          // batch stride of ss_in and ss_out (floats)
  float norm_eps, inv_feat;  // eps, 1 / (H P)
  unsigned long long* trace;  // diagnostics: per-sub-chunk event clocks of CTA 0, then
                              // [start ns, end ns, SM] of every CTA; or NULL
  int withhold_loads;         // self-test of the timeout path: issue no TMA loads, so
                              // every wait on them runs out (0 in every other launch)
};

// Trace events (clock64 of CTA 0), one row of kTraceEvents per sub-chunk.
enum {
  EV_LOADS = 0, EV_S_ISSUED, EV_C_ISSUED, EV_MASK_START, EV_MASK_DONE, EV_LAM_READY, EV_XP_DONE, EV_C_SEEN,
  EV_STATE_PUB, EV_EPI_DONE, EV_C_READY, EV_C_MID, EV_S_READY, EV_MASK_LD, EV_MASK_B01, EV_MASK_LD2,
  EV_MASK_B23, EV_MASK_WST, kTraceEvents = 24
};

// barrier indices
enum {
  FULL0 = 0, EMPTY0 = 2, SFULL0 = 4, PFULL0 = 6, CFULL0 = 8, TEMPTY0 = 10, STATEFULL = 12, DRAIN = 13, LAMRDY0 = 14,
  YFREE0 = 18,  // [X' buffer]: the y tile staged there has been read by its TMA store
  XFULL0 = 20   // [TMEM buffer]: the sub-chunk's x tile copied into its columns 0-31
};
constexpr int AUX = 64;  // threads of warps 0-1
// Warp w runs on SM sub-partition w % 4 and may only touch TMEM lane quarter
// w % 4, so the rows with the most mask work (quarter 3) share a sub-partition
// with the lightest single-thread role.
constexpr int W_TMA = 2, W_MMA = 3;

struct Ctl {
  uint64_t* bar;
  volatile int* abort;
  // Sleeps in mbarrier.try_wait (hinted) and reads the timer only every 32
  // probes, so waiting warps take almost no issue slots from working ones.
  __device__ bool wait(int i, uint32_t parity) const {
    if (*abort) return false;
    uint64_t* b = bar + i;
    if (mbar_try_wait(b, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t spin = 1;; ++spin) {
      if (mbar_try_wait_sleep(b, parity, 20000u)) return true;
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
};

__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n)); }

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
// 2^x with the ex2.approx PTX instruction (flushes denormals; |rel err| ~ 2^-22).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
constexpr float kLog2e = 1.4426950408889634f;

// Packed fp32x2 arithmetic (sm_100): two lanes of fp32 per instruction, each
// lane rounded like the scalar operation.
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

__device__ __forceinline__ float2 bf2_to_f2(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

// XDT: the dt-scaled input variant; NORM: a layer of a stack with the RMS norm
// fused (input scaled from ss_in when given, sums of squares to ss_out when
// given); MULTI: the chunk-scan step with cpc consecutive chunks per CTA, each
// started from its given state.  Separate instantiations, so that the plain
// scan carries none of their per-column factors, sums and reloads.
template <bool XDT, bool NORM, bool MULTI = false>
__global__ void __launch_bounds__(THREADS, 1)
    k_ssd_fused(Params p, const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_b,
                const __grid_constant__ CUtensorMap map_c, const __grid_constant__ CUtensorMap map_y) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the __shared__ array by an offset so
  // the compiler keeps the shared address space (LDS/STS, not generic access)
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(sm);
  float* lamb = reinterpret_cast<float*>(sm + OFF_LAM);
  float* ecolb = reinterpret_cast<float*>(sm + OFF_ECOL);
  float* dtsb = reinterpret_cast<float*>(sm + OFF_DTS);
  float* rnb = reinterpret_cast<float*>(sm + OFF_RN);
  constexpr bool CF = XDT || NORM;  // the input term has a factor per column s
  float* wtot = reinterpret_cast<float*>(sm + OFF_WTOT);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(sm + OFF_MISC + 4);
  Ctl ctl{bar, abort_flag};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool chunked = p.mode != MODE_SCAN && (int64_t)blockIdx.x >= p.whole;
  const int64_t cb = (int64_t)blockIdx.x - p.whole;                // chunk CTA index (step modes)
  const int64_t bh = chunked ? p.seq0 + cb % p.nseq : (int64_t)blockIdx.x;
  // chunk of this CTA (step modes; MULTI: its first of cpc)
  const int64_t cidx = chunked ? (MULTI ? cb / p.nseq * p.cpc : cb / p.nseq) : 0;
  const int b = (int)(bh / p.H), h = (int)(bh % p.H);
  const int g = h / (p.H / p.G);
  const int t_base = (int)(cidx * p.Q);                          // first token of this CTA
  const int nsub = chunked ? (int)ceil_div(min((MULTI ? p.cpc : 1) * p.Q, p.L - t_base), (int64_t)T) : p.nsub;
  const int64_t cslot = (bh - p.seq0) * p.nc + cidx;            // chunk slot (step modes)
  const float* init_ptr = chunked ? (p.mode == MODE_CHUNK_SCAN ? p.chunk_init + cslot * NS * P : nullptr)
                                  : (p.init ? p.init + bh * NS * P : nullptr);
  float* final_ptr = chunked ? (p.mode == MODE_CHUNK_STATE ? p.chunk_final + cslot * NS * P : nullptr)
                             : (p.final_state ? p.final_state + bh * NS * P : nullptr);
  unsigned long long* const trace = (p.trace && blockIdx.x == 0) ? p.trace : nullptr;
  auto mark = [&](int j, int ev) {
    if (trace) trace[j * kTraceEvents + ev] = clock64();
  };
  unsigned long long* const cta_rec =
      p.trace ? p.trace + (int64_t)p.nsub * kTraceEvents + 3 * (int64_t)blockIdx.x : nullptr;
  if (cta_rec && threadIdx.x == 0) {
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    cta_rec[0] = globaltimer_ns();
    cta_rec[2] = smid;
  }

  if (warp == W_MMA) tmem_alloc(tmem_slot, TMEM_COLS);
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[FULL0 + i], 1);
      mbar_init(&bar[EMPTY0 + i], 1);
      mbar_init(&bar[SFULL0 + i], 1);
      mbar_init(&bar[PFULL0 + i], T + AUX);
      mbar_init(&bar[CFULL0 + i], 1);
      mbar_init(&bar[TEMPTY0 + i], T);
      mbar_init(&bar[YFREE0 + i], 1);
      mbar_init(&bar[XFULL0 + i], 1);
    }
    mbar_init(&bar[STATEFULL], T);
    mbar_init(&bar[DRAIN], 1);
    for (int i = 0; i < 4; ++i) mbar_init(&bar[LAMRDY0 + i], AUX);
    fence_mbar_init();
    prefetch_tmap(&map_x);
    prefetch_tmap(&map_b);
    prefetch_tmap(&map_c);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == W_TMA) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // L2 prefetch runs kPrefetch sub-chunks ahead of the shared-memory loads,
      // so a stage freed by the products of sub-chunk j-2 refills from L2
      constexpr int kPrefetch = 3;
      auto prefetch = [&](int jp) {
        if (jp >= nsub) return;
        const int tp = t_base + jp * T;
        tma_prefetch_4d(&map_x, 0, h, tp, b);
        tma_prefetch_4d(&map_b, 0, g, tp, b);
        tma_prefetch_4d(&map_b, 64, g, tp, b);
        tma_prefetch_4d(&map_c, 0, g, tp, b);
        tma_prefetch_4d(&map_c, 64, g, tp, b);
      };
      for (int jp = 0; jp < kPrefetch; ++jp) prefetch(jp);
      const int nload = nsub & (p.withhold_loads - 1);  // 0 or nsub (withhold_loads is 0 or 1)
      int issued = 0;
      for (int j = 0; j < nload; ++j) {
        const int st = j & 1;
        prefetch(j + kPrefetch);
        if (j >= 2 && !ctl.wait(EMPTY0 + st, ((j >> 1) + 1) & 1)) break;
        uint8_t* sx = sm + st * STAGE;
        const int t0 = t_base + j * T;
        mbar_arrive_expect_tx(&bar[FULL0 + st], TX_BYTES);
        tma_load_4d(sx + OFF_X, &map_x, &bar[FULL0 + st], 0, h, t0, b);
        tma_load_4d(sx + OFF_B, &map_b, &bar[FULL0 + st], 0, g, t0, b);
        tma_load_4d(sx + OFF_B + TILE, &map_b, &bar[FULL0 + st], 64, g, t0, b);
        tma_load_4d(sx + OFF_C, &map_c, &bar[FULL0 + st], 0, g, t0, b);
        tma_load_4d(sx + OFF_C + TILE, &map_c, &bar[FULL0 + st], 64, g, t0, b);
        issued = j + 1;
        mark(j, EV_LOADS);
      }
      // drain: the last loads issued to each stage must land before the CTA may
      // exit (also after an early exit from the loop)
      for (int j = (issued > 2 ? issued - 2 : 0); j < issued; ++j) {
        uint64_t* fb = &bar[FULL0 + (j & 1)];
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(fb, (j >> 1) & 1) && globaltimer_ns() - t0 < 1000000000ull) {
        }
      }
    }
  } else if (warp == W_MMA) {
    // ------------------------------------------------------------ MMA issuer
    // Polls three queues and issues whichever is ready: the products c(jc) of
    // sub-chunk jc (on the state's critical path, checked first), the copy of
    // the x tile of sub-chunk jx into TMEM for the epilogue's skip term, and
    // S(js) of a later sub-chunk.  S(js) needs its stage loaded and its TMEM
    // buffer released by the epilogue of js-2; c(jc) needs P and X' (PFULL) and
    // the bf16 state b(jc-1) (STATEFULL); the copy goes over P's first 32
    // columns, so it waits for the products of jx to complete (an MMA and a
    // later tcgen05.cp of one thread are not ordered by the pipe), and the
    // stage of jx is released only after it.
    if (lane == 0) {
      const uint32_t idS = idesc_bf16(128, 128, false, false);
      const uint32_t idY = idesc_bf16(128, 64, false, true);
      const uint32_t idB = idesc_bf16(128, 64, true, true);
      // Descriptors of stage 0, computed once: each MMA only advances the start
      // address (one 64-bit add on the issuing thread's critical path).
      const uint64_t dC = smem_desc(sbase + OFF_C, 16, 1024);      // K-major (A of S and y_inter)
      const uint64_t dBk = smem_desc(sbase + OFF_B, 16, 1024);     // K-major (B of S)
      const uint64_t dBmn = smem_desc(sbase + OFF_B, TILE, 1024);  // MN-major (A of b_intra)
      const uint64_t dX = smem_desc(sbase + OFF_X, TILE, 1024);    // MN-major (B of y_intra)
      const uint64_t dXp = smem_desc(sbase + OFF_XP, TILE, 1024);  // MN-major (B of b_intra)
      const uint64_t dPrev = smem_desc(sbase + OFF_PREV, TILE, 1024);
      const uint64_t dXk = smem_desc(sbase + OFF_X, 16, 1024);     // K-major rows (the copy's source)
      int js = 0, jc = 0, jx = 0;
      uint32_t idle = 0;
      uint64_t t_last = globaltimer_ns();
      while (jx < nsub) {
        bool progress = false;
        if (jc < js && mbar_test_wait(&bar[PFULL0 + (jc & 1)], (jc >> 1) & 1) &&
            mbar_test_wait(&bar[STATEFULL], jc & 1)) {
          const int st = jc & 1, buf = jc & 1;
          mark(jc, EV_C_READY);
          tc_fence_after();
          const uint32_t base = tmem + buf * 256;
          const uint64_t cB = desc_advance(dBmn, st * STAGE), cXp = desc_advance(dXp, (jc & 1) * TILE);
          const uint64_t cX = desc_advance(dX, st * STAGE), cC = desc_advance(dC, st * STAGE);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)  // b_intra = B^T X'  (the state chain needs it first)
            mma_ss(base + 192, desc_advance(cB, ks * 2048), desc_advance(cXp, ks * 2048), idB, ks > 0);
          mark(jc, EV_C_MID);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)  // y_intra = P X
            mma_ts(base + 128, base + ks * 8, desc_advance(cX, ks * 2048), idY, ks > 0);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)  // y_inter = C prev  (K = dstate)
            mma_ss(base + 64, desc_advance(cC, (ks >> 2) * TILE + (ks & 3) * 32), desc_advance(dPrev, ks * 2048), idY,
                   ks > 0);
          mma_commit(&bar[CFULL0 + buf]);
          mark(jc, EV_C_ISSUED);
          ++jc;
          progress = true;
        }
        if (jx < jc && mbar_test_wait(&bar[CFULL0 + (jx & 1)], (jx >> 1) & 1)) {
          const int st = jx & 1, buf = jx & 1;
          tc_fence_after();
          const uint64_t xs = desc_advance(dXk, st * STAGE);
#pragma unroll
          for (int k = 0; k < 4; ++k)  // x row t -> lane t, bf16 pairs in columns 8k .. 8k+7
            tmem_cp_128x256b(tmem + buf * 256 + 8 * k, desc_advance(xs, k * 32));
          mma_commit(&bar[XFULL0 + buf]);
          mma_commit(&bar[EMPTY0 + st]);
          ++jx;
          progress = true;
        }
        if (js < nsub && mbar_test_wait(&bar[FULL0 + (js & 1)], (js >> 1) & 1) &&
            (js < 2 || mbar_test_wait(&bar[TEMPTY0 + (js & 1)], ((js >> 1) + 1) & 1))) {
          const int st = js & 1, buf = js & 1;
          mark(js, EV_S_READY);
          tc_fence_after();
          const uint32_t tS = tmem + buf * 256;
          const uint64_t sCd = desc_advance(dC, st * STAGE), sBd = desc_advance(dBk, st * STAGE);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t koff = (ks >> 2) * TILE + (ks & 3) * 32;
            mma_ss(tS, desc_advance(sCd, koff), desc_advance(sBd, koff), idS, ks > 0);
          }
          mma_commit(&bar[SFULL0 + buf]);
          mark(js, EV_S_ISSUED);
          ++js;
          progress = true;
        }
        if (progress) {
          idle = 0;
        } else if ((++idle & 63) == 0) {
          const uint64_t now = globaltimer_ns();
          if (idle == 64) t_last = now;
          if (*abort_flag) break;
          if (now - t_last > 1000000000ull) {
            *abort_flag = 1;
            atomicExch(&g_device_status, 2);
            break;
          }
        } else {
          __nanosleep(20);
        }
      }
      // every MMA issued must complete before TMEM is released (also on abort)
      mma_commit(&bar[DRAIN]);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&bar[DRAIN], 0) && globaltimer_ns() - t0 < 1000000000ull) {
      }
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ dt, lam, decay factors, X'
    const int a = threadIdx.x;  // 0..63 (warps 0-1)
    // lam comes from dt (whole scan, and step modes without a step-1 output)
    // or from step 1's output (lamc)
    const float* lamc = (chunked && p.lam_in) ? p.lam_in + cslot * p.Q : nullptr;
    const float Ah = lamc ? 0.f : p.A[h];
    const float* dtb = p.dt + (int64_t)b * p.sdt + h;
    auto load_dt = [&](int j, float& d0, float& d1) {
      const int64_t t0 = (int64_t)t_base + (int64_t)j * T + 2 * a;
      d0 = (!lamc && j < nsub && t0 < p.L) ? dtb[t0 * p.lddt] : 0.f;
      d1 = (!lamc && j < nsub && t0 + 1 < p.L) ? dtb[(t0 + 1) * p.lddt] : 0.f;
    };
    // r of tokens 2a, 2a+1 of sub-chunk j from the H per-head sums of squares
    // of the previous layer's stored y (0 past L).  A token's H sums are
    // contiguous.  With H % 4 == 0 the first 32 of them (8 float4 per token)
    // are loaded one sub-chunk ahead into registers (issue_rn) and summed when
    // needed (finish_rn), so the trip to L2 overlaps a whole iteration; sums
    // past the first 32 heads, and rows with H % 4 != 0, are loaded when needed.
    const bool vec = (p.H & 3) == 0;
    float4 pv[8], pw[8];
    auto rn_row = [&](int j, int k) { return p.ss_in + (int64_t)b * p.sss + ((int64_t)j * T + 2 * a + k) * p.H; };
    auto issue_rn = [&](int j) {
      const int64_t t0 = (int64_t)j * T + 2 * a;
      const bool use = p.ss_in && vec && j < nsub;
      const float4* q0 = use ? reinterpret_cast<const float4*>(rn_row(j, 0)) : nullptr;
      const float4* q1 = use ? reinterpret_cast<const float4*>(rn_row(j, 1)) : nullptr;
      const int n4 = p.H >> 2;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        pv[i] = (use && i < n4 && t0 < p.L) ? q0[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        pw[i] = (use && i < n4 && t0 + 1 < p.L) ? q1[i] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    };
    auto finish_rn = [&](int j, float& r0, float& r1) {
      if (!p.ss_in) {  // the stack's first layer: its input is used as is
        r0 = r1 = 1.f;
        return;
      }
      const int64_t t0 = (int64_t)j * T + 2 * a;
      const bool in0 = t0 < p.L, in1 = t0 + 1 < p.L;
      float s0 = 0.f, s1 = 0.f;
      if (vec) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {  // the prefetched first 32 heads
          s0 += (pv[i].x + pv[i].y) + (pv[i].z + pv[i].w);
          s1 += (pw[i].x + pw[i].y) + (pw[i].z + pw[i].w);
        }
        const float4* q0 = reinterpret_cast<const float4*>(rn_row(j, 0));
        const float4* q1 = reinterpret_cast<const float4*>(rn_row(j, 1));
        const int n4 = p.H >> 2;
        for (int i0 = 8; i0 < n4; i0 += 8) {  // heads past the first 32
          float4 v[8], w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const bool ok = i0 + i < n4;
            v[i] = (ok && in0) ? q0[i0 + i] : make_float4(0.f, 0.f, 0.f, 0.f);
            w[i] = (ok && in1) ? q1[i0 + i] : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            s0 += (v[i].x + v[i].y) + (v[i].z + v[i].w);
            s1 += (w[i].x + w[i].y) + (w[i].z + w[i].w);
          }
        }
      } else {
        const float* q = rn_row(j, 0);
        for (int i0 = 0; i0 < p.H; i0 += 16) {
          float v[16], w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const bool ok = i0 + i < p.H;
            v[i] = (ok && in0) ? q[i0 + i] : 0.f;
            w[i] = (ok && in1) ? q[p.H + i0 + i] : 0.f;
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            s0 += v[i];
            s1 += w[i];
          }
        }
      }
      r0 = in0 ? rsqrtf(s0 * p.inv_feat + p.norm_eps) : 0.f;
      r1 = in1 ? rsqrtf(s1 * p.inv_feat + p.norm_eps) : 0.f;
    };
    float d0, d1;  // dt of the next sub-chunk to be tabled (tokens 2a, 2a+1)
    load_dt(0, d0, d1);
    if constexpr (NORM) issue_rn(0);
    // The tables of sub-chunk jt into slot jt & 3 (lam, the column decays and
    // factors, r), then LAMRDY; dt and the norm sums of jt + 1 are requested on
    // the way.  The loop below runs them one sub-chunk ahead of X', so the
    // mask never waits for the X' of the sub-chunk before it.
    auto tables = [&](int jt) {
      const int slot = jt & 3;
      float n0, n1;
      load_dt(jt + 1, n0, n1);
      // inclusive scan of dt*A over the 128 tokens (two per thread)
      const float l0 = d0 * Ah, l1 = d1 * Ah;
      float v = l0 + l1;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float nb = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += nb;
      }
      if (lane == 31) wtot[warp] = v;
      named_sync(1, AUX);
      const float pre = (warp == 1) ? wtot[0] : 0.f;
      float lam1 = v + pre;       // token 2a+1
      float lam0 = lam1 - l1;     // token 2a
      if (lamc) {                 // step modes: sub-chunk-local sums from step 1's output
        const float* ls = lamc + jt * T;  // chunks of one sequence are contiguous in step 1's output
        bool chunk_start = jt == 0;
        if constexpr (MULTI) chunk_start = (jt * T) % p.Q == 0;
        const float base0 = chunk_start ? 0.f : ls[-1];
        lam0 = ls[2 * a] - base0;
        lam1 = ls[2 * a + 1] - base0;
      }
      // lam is kept in log2 units (lam * log2 e) so every decay is one ex2
      float* lj = lamb + slot * T;
      float* ec = ecolb + slot * T;
      float* dts = dtsb + slot * T;
      lj[2 * a] = lam0 * kLog2e;
      lj[2 * a + 1] = lam1 * kLog2e;
      // the input term's factor per column s: dt_s (dt-scaled input) times r_s
      // (normalised input)
      float cf0 = 1.f, cf1 = 1.f;
      if constexpr (XDT) {
        cf0 = d0;
        cf1 = d1;
      }
      if constexpr (NORM) {
        float rn0, rn1;
        finish_rn(jt, rn0, rn1);
        rnb[slot * T + 2 * a] = rn0;
        rnb[slot * T + 2 * a + 1] = rn1;
        cf0 *= rn0;
        cf1 *= rn1;
      }
      if constexpr (CF) {
        dts[2 * a] = cf0;
        dts[2 * a + 1] = cf1;
      }
      named_sync(1, AUX);
      // decay from each column s to the last column of its 32-block (times the
      // column's input factor, which every product with column s carries)
      const float lr = lj[(2 * a) | 31];
      ec[2 * a] = ex2(lr - lj[2 * a]);
      ec[2 * a + 1] = ex2(lr - lj[2 * a + 1]);
      if constexpr (CF) {
        ec[2 * a] *= cf0;
        ec[2 * a + 1] *= cf1;
      }
      mbar_arrive(&bar[LAMRDY0 + slot]);
      if (a == 0) mark(jt, EV_LAM_READY);
      d0 = n0;
      d1 = n1;
      if constexpr (NORM) issue_rn(jt + 1);  // in flight until the next tables
    };
    tables(0);
    for (int j = 0; j < nsub; ++j) {
      const int st = j & 1, slot = j & 3;
      // Slot (j + 1) & 3 last held sub-chunk j - 3, whose readers (its mask,
      // epilogue and X') are done: this loop waited for its products and its y
      // store in iteration j - 1.
      if (j + 1 < nsub) tables(j + 1);
      const float* lj = lamb + slot * T;
      const float* dts = dtsb + slot * T;
      // X'_j = diag(exp(lam_end - lam_t)) X_j, rows a and a + 64, into buffer j & 1
      // (free once the products of sub-chunk j - 2 have completed and its y tile,
      // staged in the same buffer, has been read by the TMA store)
      bool ok = ctl.wait(FULL0 + st, (j >> 1) & 1);
      if (ok && j >= 2) ok = ctl.wait(CFULL0 + st, ((j - 2) >> 1) & 1);
      if (ok && j >= 2) ok = ctl.wait(YFREE0 + st, ((j - 2) >> 1) & 1);  // y(j-2) staged here is stored
      if (ok) {
        const float lam_end = lj[T - 1];  // log2 units
        const uint4* src = reinterpret_cast<const uint4*>(sm + st * STAGE + OFF_X);
        uint4* dst = reinterpret_cast<uint4*>(sm + OFF_XP + st * TILE);
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int row = a + 64 * rr;
          float w = ex2(lam_end - lj[row]);
          if constexpr (CF) w *= dts[row];
          uint4 v4[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) v4[c] = src[swz128(row, c * 8) >> 4];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t* u = reinterpret_cast<uint32_t*>(&v4[c]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {  // fp32 product, one rounding (the state accumulates it)
              const float2 f = mul2(bf2_to_f2(u[i]), make_float2(w, w));
              u[i] = pack_bf16(f.x, f.y);
            }
            dst[swz128(row, c * 8) >> 4] = v4[c];
          }
        }
        fence_async_smem();
      }
      mbar_arrive(&bar[PFULL0 + st]);
      if (a == 0) mark(j, EV_XP_DONE);
      named_sync(1, AUX);  // wtot reuse
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ P = S (.) L
    const int q = warp & 3;          // TMEM lane quarter = 32-row block
    const int row = q * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
    for (int j = 0; j < nsub; ++j) {
      const int buf = j & 1, slot = j & 3;
      bool ok = ctl.wait(LAMRDY0 + slot, (j >> 2) & 1);
      if (ok) ok = ctl.wait(SFULL0 + buf, (j >> 1) & 1);
      tc_fence_after();
      if (q == 3 && lane == 0) mark(j, EV_MASK_START);
      const float* lj = lamb + slot * T;   // log2 units
      const float* ec = ecolb + slot * T;
      const float lam_t = lj[row];
      const uint32_t tS = tl + buf * 256;
      const float4* ec4 = reinterpret_cast<const float4*>(ec);
      const float4* lj4 = reinterpret_cast<const float4*>(lj);
      const float4* dt4 = reinterpret_cast<const float4*>(dtsb + slot * T);
      // P block kb (32 columns) of this row from the S values r[0..31]
      auto make_block = [&](int kb, const uint32_t* r, uint32_t* pk) {
        if (kb < q) {
          // below the diagonal block: exp(lam_t - lam_s) = 2^(lt - l_end(kb)) * ec[s]
          const float rowf = ex2(lam_t - lj[32 * kb + 31]);
          const float2 rf2 = make_float2(rowf, rowf);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const float4 c = ec4[8 * kb + v];
            const float2 a = mul2(mul2(make_float2(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1])),
                                       make_float2(c.x, c.y)), rf2);
            const float2 bb = mul2(mul2(make_float2(__uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3])),
                                        make_float2(c.z, c.w)), rf2);
            pk[2 * v] = pack_bf16(a.x, a.y);
            pk[2 * v + 1] = pack_bf16(bb.x, bb.y);
          }
        } else if (kb == q) {
          // diagonal block: direct decays, clamped at 0 above the diagonal and then zeroed
          const int rl = row - 32 * kb;  // column index of the diagonal within the block
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const float4 l = lj4[8 * kb + v];
            float e0 = ex2(fminf(lam_t - l.x, 0.f)), e1 = ex2(fminf(lam_t - l.y, 0.f));
            float e2 = ex2(fminf(lam_t - l.z, 0.f)), e3 = ex2(fminf(lam_t - l.w, 0.f));
            if constexpr (CF) {  // the columns' input factors
              const float4 fx = dt4[8 * kb + v];
              e0 *= fx.x; e1 *= fx.y; e2 *= fx.z; e3 *= fx.w;
            }
            const float f0 = (4 * v + 0 <= rl) ? __uint_as_float(r[4 * v + 0]) * e0 : 0.f;
            const float f1 = (4 * v + 1 <= rl) ? __uint_as_float(r[4 * v + 1]) * e1 : 0.f;
            const float f2 = (4 * v + 2 <= rl) ? __uint_as_float(r[4 * v + 2]) * e2 : 0.f;
            const float f3 = (4 * v + 3 <= rl) ? __uint_as_float(r[4 * v + 3]) * e3 : 0.f;
            pk[2 * v] = pack_bf16(f0, f1);
            pk[2 * v + 1] = pack_bf16(f2, f3);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = 0u;
        }
      };
      // One 32-column block per TMEM round trip (load, wait, form, store): with
      // two blocks per round trip, or the next block's load left in flight while
      // this one is formed, the headline scan measured 6 % and 30 % slower.
#pragma unroll 1
      for (int kb = 0; kb < 4; ++kb) {
        uint32_t r0[32], pk[16];
        // warp-uniform: only blocks on or below the diagonal block are read
        if (kb <= q) {
          tmem_ld32(tS + 32 * kb, r0);
          tmem_wait_ld();
        }
        if (q == 3 && lane == 0 && (kb & 1) == 0) mark(j, kb == 0 ? EV_MASK_LD : EV_MASK_LD2);
        make_block(kb, r0, pk);
        tmem_st16(tS + 16 * kb, pk);
        if (q == 3 && lane == 0 && (kb & 1) == 1) mark(j, kb == 1 ? EV_MASK_B01 : EV_MASK_B23);
      }
      tmem_wait_st();
      if (q == 3 && lane == 0) mark(j, EV_MASK_WST);
      tc_fence_before();
      (void)ok;
      mbar_arrive(&bar[PFULL0 + buf]);
      if (q == 3 && lane == 0) mark(j, EV_MASK_DONE);
    }
  } else {
    // ------------------------------------------------------------ y, state, final
    const int q = warp & 3;
    const int r = q * 32 + lane;  // state row n and output row t
    const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
    const float Dh = p.D ? p.D[h] : 0.f;
    // x of each sub-chunk comes from TMEM: the issuer copies the stage's x
    // tile there once the products are done (the skip term D x_t)
    float s[P];
    if (chunked) grid_dep_wait();  // start states from the kernel before (a programmatic launch)
    if (init_ptr) {
      const float4* src = reinterpret_cast<const float4*>(init_ptr + (int64_t)r * P);
#pragma unroll
      for (int i = 0; i < P / 4; ++i) {
        const float4 v = src[i];
        s[4 * i] = v.x; s[4 * i + 1] = v.y; s[4 * i + 2] = v.z; s[4 * i + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < P; ++i) s[i] = 0.f;
    }
    const uint32_t sPrev = sbase + OFF_PREV;
    auto publish_state = [&]() {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 v;
        v.x = pack_bf16(s[8 * c + 0], s[8 * c + 1]);
        v.y = pack_bf16(s[8 * c + 2], s[8 * c + 3]);
        v.z = pack_bf16(s[8 * c + 4], s[8 * c + 5]);
        v.w = pack_bf16(s[8 * c + 6], s[8 * c + 7]);
        sts128(sPrev + swz128(r, 8 * c), v);
      }
      fence_async_smem();
      mbar_arrive(&bar[STATEFULL]);
    };
    publish_state();
    for (int j = 0; j < nsub; ++j) {
      const int buf = j & 1;
      bool ok = ctl.wait(CFULL0 + buf, (j >> 1) & 1);
      if (ok) ok = ctl.wait(LAMRDY0 + (j & 3), (j >> 2) & 1);      // acquire lam of this sub-chunk
      tc_fence_after();
      if (r == 0) mark(j, EV_C_SEEN);
      const float* lj = lamb + (j & 3) * T;
      const float lam_end = lj[T - 1];
      const uint32_t base = tl + buf * 256;
      // state: s_j = exp(lam_end) s_{j-1} + b_intra
      const float dec = ex2(lam_end);  // lam in log2 units
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t v[32];
        tmem_ld32(base + 192 + 32 * c, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 o = fma2(make_float2(dec, dec), make_float2(s[32 * c + i], s[32 * c + i + 1]),
                                make_float2(__uint_as_float(v[i]), __uint_as_float(v[i + 1])));
          s[32 * c + i] = o.x;
          s[32 * c + i + 1] = o.y;
        }
      }
      if constexpr (MULTI) {
        // the next sub-chunk starts a chunk: its products take that chunk's given
        // state, not this running one (y of this sub-chunk does not use it)
        if (j + 1 < nsub && ((int64_t)(j + 1) * T) % p.Q == 0) {
          const float4* src = reinterpret_cast<const float4*>(
              p.chunk_init + (cslot + (int64_t)(j + 1) * T / p.Q) * NS * P + (int64_t)r * P);
#pragma unroll
          for (int i = 0; i < P / 4; ++i) {
            const float4 v = src[i];
            s[4 * i] = v.x; s[4 * i + 1] = v.y; s[4 * i + 2] = v.z; s[4 * i + 3] = v.w;
          }
        }
      }
      if (ok) publish_state();
      if (r == 0) mark(j, EV_STATE_PUB);
      if (ok) ok = ctl.wait(XFULL0 + buf, (j >> 1) & 1);  // x of this sub-chunk in TMEM
      tc_fence_after();
      // y_t = y_intra + exp(lam_t) y_inter + D x_t, staged as a 128-B-swizzled tile
      // in the X' buffer of this sub-chunk (free: its products have completed) and
      // written by one TMA store, coalesced, rows past L clipped by the copy.  Per-
      // row global stores (32 rows 10 KB apart per warp instruction) held up the
      // masking warps' shared-memory loads in the same memory pipe.
      const float et = ex2(lj[r]);
      const uint32_t ystage = sbase + OFF_XP + buf * TILE;
      // the skip term sees the input as the scan does: r_t x_t when normalised
      float Dt = Dh;
      if constexpr (NORM) Dt *= rnb[(j & 3) * T + r];
      float ss = 0.f;  // sum of squares of the stored (bf16) y row
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t yi[16], ye[16], xr[8];
        tmem_ld16(base + 128 + 16 * c, yi);
        tmem_ld16(base + 64 + 16 * c, ye);
        tmem_ld8(base + 8 * c, xr);
        tmem_wait_ld();
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int cc = 2 * c + h2;  // 8-column chunk
          const uint32_t* xu = xr + 4 * h2;
          uint4 ov;
          uint32_t* o = reinterpret_cast<uint32_t*>(&ov);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int k0 = h2 * 8 + 2 * i;
            const float2 xf = bf2_to_f2(xu[i]);
            float2 yo = fma2(make_float2(Dt, Dt), xf, make_float2(__uint_as_float(yi[k0]), __uint_as_float(yi[k0 + 1])));
            yo = fma2(make_float2(et, et), make_float2(__uint_as_float(ye[k0]), __uint_as_float(ye[k0 + 1])), yo);
            o[i] = pack_bf16(yo.x, yo.y);
            if constexpr (NORM) {
              const float2 q = bf2_to_f2(o[i]);
              ss = fmaf(q.x, q.x, ss);
              ss = fmaf(q.y, q.y, ss);
            }
          }
          sts128(ystage + swz128(r, 8 * cc), ov);
        }
      }
      if (NORM && p.ss_out) {  // this head's share of the next layer's RMS norm
        const int64_t tg = (int64_t)t_base + (int64_t)j * T + r;
        if (tg < p.L) p.ss_out[(int64_t)b * p.sss + tg * p.H + h] = ss;
      }
      tc_fence_before();
      mbar_arrive(&bar[TEMPTY0 + buf]);
      fence_async_smem();
      named_sync(2, T);  // the 128 rows are staged
      if (r == 0) {
        if (p.y) {
          tma_store_4d(&map_y, sm + OFF_XP + buf * TILE, 0, h, t_base + j * T, b);
          tma_store_commit();
          tma_store_wait_read0();
        }
        mbar_arrive(&bar[YFREE0 + buf]);
      }
      if (r == 0) mark(j, EV_EPI_DONE);
    }
    if (r == 0) tma_store_wait0();  // the y tiles are in global memory before the CTA exits
    if (final_ptr) {
      float4* dst = reinterpret_cast<float4*>(final_ptr + (int64_t)r * P);
#pragma unroll
      for (int i = 0; i < P / 4; ++i) dst[i] = make_float4(s[4 * i], s[4 * i + 1], s[4 * i + 2], s[4 * i + 3]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
    tmem_relinquish();
  }
  if (cta_rec && threadIdx.x == 0) cta_rec[1] = globaltimer_ns();
}

}  // namespace fused

bool fused_supported(const Problem& p) {
  return p.io == SSD_BF16 && p.P == fused::P && p.N == fused::NS && p.Q % fused::T == 0 && p.B * p.H < (1ll << 31);
}

bool tc_supported(const Problem& p) { return fused_supported(p) && p.B * p.H * p.nc < (1ll << 31); }


bool uses_pair_kernel(const Problem& p) { return p.two_heads && pair_supported(p); }

// Segments, where one CTA per (batch, head) sequence would leave SMs idle:
// with fewer sequences than SMs, or with B*H = q*SMs + r sequences whose last
// r run as a partial round of CTAs while the other SMs have nothing left.
// The first `whole` sequences run whole (one CTA each); every later one is
// cut into nseg segments of qseg tokens (the page's chunk decomposition one
// level up, "分块推理…" §2.1-§2.2, with a segment as the chunk).  Three launches:
// k_ssd_segment_states (csrc/ssd_lean.cu) forms each segment's end state from
// a zero start and its total log-decay, k_state_passing combines them in order into each
// segment's start state (and the sequence's final state), and the full
// kernel runs the whole sequences first and then every segment from its
// start state, so the short segment CTAs fill the SMs that the last whole
// ones leave free.  Chosen only where a cost model of CTA rounds (a segment's
// end state costing about a third of its full scan) predicts a gain.
struct SegPlan {
  int nseg;       // 1: whole sequences in one launch
  int64_t qseg;   // segment length in tokens (a multiple of 128)
  int64_t whole;  // sequences 0..whole-1 run whole; the rest are segmented
};
static int g_fused_segments = 0;         // forced by a self-test (0: the cost model decides)
static int64_t g_fused_whole = 0;        // sequences run whole when the segment count is forced
void set_fused_segments(int nseg) { set_fused_split(nseg, 0); }
void set_fused_split(int nseg, int64_t whole) {
  g_fused_segments = nseg > 0 ? nseg : 0;
  g_fused_whole = whole > 0 ? whole : 0;
}

// Finish time, in sub-chunk periods, of `nw` CTAs of cost w followed by `ns`
// CTAs of cost s on `nsm` SMs, each CTA starting on the SM that frees first
// (CTAs start in grid order).
static double makespan(int64_t nsm, int64_t nw, double w, int64_t ns, double s) {
  const int64_t q = nw / nsm, r = nw % nsm;  // r SMs run one more whole CTA
  const double t0 = q * w, t1 = t0 + w;
  const int64_t a = nsm - r;                // SMs free at t0
  if (r == 0) return t0 + (double)ceil_div(ns, nsm) * s;
  // segments first go to the a SMs free at t0, until those pass t1 ...
  const int64_t m = (int64_t)std::ceil(w / s);
  if (ns <= a * m) return std::max(t1, t0 + (double)ceil_div(ns, a) * s);
  // ... then to every SM in turn, the r SMs free at t1 first
  const int64_t n2 = ns - a * m, k = n2 / nsm, e = n2 % nsm;
  return std::max(t0 + (m + k + (e > r ? 1 : 0)) * s, t1 + (k + (e > 0 ? 1 : 0)) * s);
}

static SegPlan seg_plan(const Problem& p) {
  const int64_t nsub = ceil_div(p.L, (int64_t)fused::T), bh = p.B * p.H;
  SegPlan plan{1, 0, bh};
  if (uses_pair_kernel(p) || !fused_supported(p)) return plan;
  const int64_t nsm = split::sm_count();
  auto make = [&](int64_t n, int64_t whole) {
    const int64_t seg = ceil_div(nsub, n);
    return SegPlan{(int)ceil_div(nsub, seg), seg * fused::T, whole};
  };
  if (g_fused_segments > 0) {
    const SegPlan f = make(g_fused_segments, std::min(g_fused_whole, bh - 1));
    const bool ok = f.nseg > 1 && (bh - f.whole) * f.nseg < (1ll << 31) && (f.whole == 0 || bh - f.whole < 65536);
    return ok ? f : plan;
  }
  if (nsub < 8) return plan;
  // cost in sub-chunk periods: a CTA costs its sub-chunks plus about two of
  // pipeline fill and drain; a segment's end state about 0.35 of its scan, plus
  // one period for the combine launch
  const double w = (double)(nsub + 2);
  const double plain = (double)ceil_div(bh, nsm) * w;
  const int64_t whole = bh >= nsm ? bh - bh % nsm : 0;  // full rounds stay whole
  if (whole == bh) return plan;
  const double gain = whole > 0 ? 0.95 : 0.9;
  double best = gain * plain;
  for (int64_t n = 2; n <= 64 && n <= nsub / 4; ++n) {
    const SegPlan c = make(n, whole);
    const int64_t segs = (bh - whole) * c.nseg;
    const double seg = (double)(c.qseg / fused::T);
    const double cost = makespan(nsm, whole, w, segs, seg + 2.0) +
                        (double)ceil_div(segs, nsm) * (0.35 * seg + 1.5) + 1.0;
    if (c.nseg > 1 && segs < (1ll << 31) && cost < best) {
      best = cost;
      plan = c;
    }
  }
  return plan;
}
static size_t seg_states_bytes(const Problem& p, const SegPlan& plan) {
  const size_t states = sizeof(float) * (size_t)(p.B * p.H - plan.whole) * plan.nseg * p.N * p.P;
  return (states + 255) / 256 * 256;
}
static size_t seg_workspace_bytes(const Problem& p, const SegPlan& plan) {
  if (plan.nseg <= 1) return 0;
  return seg_states_bytes(p, plan) + sizeof(float) * (size_t)(p.B * p.H - plan.whole) * plan.nseg;
}

// Kernel launches of one fused call: three for the segmented form.
int fused_kernels_per_call(const Problem& p) { return seg_plan(p).nseg > 1 ? 3 : 1; }

// The one-head kernel keeps the running state on chip; its segmented form
// (above) needs the segments' states and decays.  The two-head kernel needs
// room for the carries of its split schedule.
size_t tc_workspace_bytes(const Problem& p) {
  if (uses_pair_kernel(p)) return pair_workspace_bytes(p);
  return seg_workspace_bytes(p, seg_plan(p));
}

// The grid of a launch: `whole` leading CTAs scan whole sequences from init
// to final_state; the step-mode CTAs cover the chunks of sequences seq0 on,
// reading start states from chunk_init or writing end states to chunk_final.
struct GridSplit {
  int64_t whole = 0, seq0 = 0;
  const float* init = nullptr;
  float* final_state = nullptr;
  bool programmatic = false;  // may start while the kernel before it finishes
  int cpc = 0;                // chunk-scan step: consecutive chunks per CTA (0: one)
};

static cudaError_t launch_mode(const Problem& p, int mode, const float* lam, const float* init, float* final_state,
                               void* y, unsigned long long* trace, cudaStream_t st, int withhold_loads = 0,
                               const NormIO* norm = nullptr, const GridSplit& split = GridSplit());

cudaError_t launch_fused_traced(const Problem& p, const float* init, float* final_state, unsigned long long* trace,
                                cudaStream_t st) {
  return launch_mode(p, fused::MODE_SCAN, nullptr, init, final_state, p.y, trace, st);
}

cudaError_t launch_fused_withheld(const Problem& p, const float* init, float* final_state, cudaStream_t st) {
  if (uses_pair_kernel(p)) return launch_pair(p, init, final_state, nullptr, 0, st, 1);
  return launch_mode(p, fused::MODE_SCAN, nullptr, init, final_state, p.y, nullptr, st, 1);
}

cudaError_t launch_fused(const Problem& p, const float* init, float* final_state, void* workspace,
                         size_t workspace_bytes, cudaStream_t st) {
  if (uses_pair_kernel(p)) return launch_pair(p, init, final_state, workspace, workspace_bytes, st, 0);
  const SegPlan plan = seg_plan(p);
  const size_t need = seg_workspace_bytes(p, plan);
  if (plan.nseg > 1 && workspace && workspace_bytes >= need) {
    Problem ps = p;  // segments as the chunks of the step modes
    ps.Q = plan.qseg;
    ps.nc = plan.nseg;
    const int64_t w = plan.whole, NP = p.N * p.P;
    float* states = static_cast<float*>(workspace);
    float* decays = reinterpret_cast<float*>(static_cast<char*>(workspace) + seg_states_bytes(p, plan));
    cudaError_t e = launch_segment_states(ps, w, states, decays, st);
    if (e != cudaSuccess) return e;
    // the combine reads one decay per segment, over the segmented sequences
    // only (with whole > 0 as one batch of B*H - whole heads, fewer than
    // 65536 by the plan)
    Problem pc = ps;
    pc.Q = 1;
    if (w > 0) {
      pc.B = 1;
      pc.H = p.B * p.H - w;
    }
    e = launch_state_passing(pc, states, decays, init ? init + w * NP : nullptr, states,
                             final_state ? final_state + w * NP : nullptr, st, /*programmatic=*/true);
    if (e != cudaSuccess) return e;
    return launch_segment_scan(ps, w, states, init, final_state, st);
  }
  return launch_mode(p, fused::MODE_SCAN, nullptr, init, final_state, p.y, nullptr, st);
}

// One layer of a stack with the RMS norm between layers fused in (one head per
// CTA): the input rows are normalised on the fly from the previous layer's
// per-(token, head) sums of squares, and this layer's sums are written for
// the next (either may be absent).
cudaError_t launch_fused_normed(const Problem& p, const float* init, float* final_state, const NormIO& norm,
                                cudaStream_t st) {
  return launch_mode(p, fused::MODE_SCAN, nullptr, init, final_state, p.y, nullptr, st, 0, &norm);
}

// The outputs of the segmented form: sequences 0..whole-1 whole (from init,
// to final_state), then every segment of the later sequences from its start
// state prev[slot] (the segments' end states come from
// launch_segment_states, csrc/ssd_lean.cu).
cudaError_t launch_segment_scan(const Problem& p, int64_t whole, const float* prev, const float* init,
                                float* final_state, cudaStream_t st) {
  GridSplit sp;
  sp.whole = whole;
  sp.seq0 = whole;
  sp.init = init;
  sp.final_state = final_state;
  sp.programmatic = true;  // its prologue and the whole sequences overlap the combine
  return launch_mode(p, fused::MODE_CHUNK_SCAN, nullptr, prev, nullptr, p.y, nullptr, st, 0, nullptr, sp);
}

// Step 4 on tensor cores: consecutive chunks of one (batch, head) per CTA,
// each started from prev[b,h,c], writing the chunks' outputs.
cudaError_t launch_chunk_scan_tc(const Problem& p, const float* lam, const float* prev, cudaStream_t st) {
  // consecutive chunks per CTA, as many as keep four CTAs per SM busy (up to
  // 16 sub-chunks): the pipeline fill of a CTA is about two sub-chunks' time
  GridSplit sp;
  sp.cpc = (int)step_chunks_per_cta(p);
  return launch_mode(p, fused::MODE_CHUNK_SCAN, lam, prev, nullptr, p.y, nullptr, st, 0, nullptr, sp);
}

static cudaError_t launch_mode(const Problem& p, int mode, const float* lam, const float* init, float* final_state,
                               void* y, unsigned long long* trace, cudaStream_t st, int withhold_loads,
                               const NormIO* norm, const GridSplit& split) {
  using namespace fused;
  // every pointer the mode reads must be present (the step entry points pass
  // only the tensors of their step)
  if (!p.x || !p.Bm) return cudaErrorInvalidValue;
  if (mode == MODE_SCAN && (!p.dt || !p.A || !p.Cm || !y)) return cudaErrorInvalidValue;
  if (mode == MODE_CHUNK_STATE && (!final_state || (!lam && (!p.dt || !p.A)))) return cudaErrorInvalidValue;
  if (mode == MODE_CHUNK_SCAN && (!init || !p.Cm || !y || (!lam && (!p.dt || !p.A)))) return cudaErrorInvalidValue;
  // the chunk-state mode never uses C: its C tiles are read from B (valid memory)
  const void* cptr = (mode == MODE_CHUNK_STATE) ? p.Bm : p.Cm;
  CUtensorMap mx, mb, mc, my;
  const uint32_t box[4] = {64, 1, (uint32_t)T, 1};
  const uint64_t dx[4] = {(uint64_t)P, (uint64_t)p.H, (uint64_t)p.L, (uint64_t)p.B};
  const uint64_t sx[3] = {(uint64_t)P * 2, (uint64_t)p.ldx * 2, (uint64_t)p.sx * 2};
  const uint64_t dbc[4] = {(uint64_t)NS, (uint64_t)p.G, (uint64_t)p.L, (uint64_t)p.B};
  const uint64_t sbc[3] = {(uint64_t)NS * 2, (uint64_t)p.ldbc * 2, (uint64_t)p.sbc * 2};
  if (!tma::encode_bf16_4d_cached(&mx, p.x, dx, sx, box) || !tma::encode_bf16_4d_cached(&mb, p.Bm, dbc, sbc, box) ||
      !tma::encode_bf16_4d_cached(&mc, cptr, dbc, sbc, box))
    return cudaErrorInvalidValue;
  if (y) {  // y has x's shape and layout, with its own batch stride
    const uint64_t sy[3] = {(uint64_t)P * 2, (uint64_t)p.ldy * 2, (uint64_t)p.sy * 2};
    if (!tma::encode_bf16_4d_cached(&my, y, dx, sy, box)) return cudaErrorInvalidValue;
  } else {
    my = mx;  // never used: no y is stored
  }
  Params kp;
  kp.mode = mode;
  kp.nc = p.nc;
  kp.Q = p.Q;
  kp.lam_in = lam;
  kp.L = p.L;
  kp.H = (int)p.H;
  kp.G = (int)p.G;
  kp.nsub = (int)ceil_div(p.L, T);
  kp.dt = p.dt;
  kp.sdt = p.sdt;
  kp.lddt = p.lddt;
  kp.input_dt = p.input_dt;
  kp.A = p.A;
  kp.D = p.D;
  // whole-sequence CTAs take init / final_state; the step modes' CTAs their
  // chunk states (mixed grids: both)
  const bool step_mode = mode != MODE_SCAN;
  kp.init = step_mode ? split.init : init;
  kp.final_state = step_mode ? split.final_state : final_state;
  kp.chunk_init = mode == MODE_CHUNK_SCAN ? init : nullptr;
  kp.chunk_final = mode == MODE_CHUNK_STATE ? final_state : nullptr;
  kp.whole = step_mode ? split.whole : 0;
  kp.seq0 = step_mode ? split.seq0 : 0;
  kp.nseq = p.B * p.H - kp.seq0;
  kp.cpc = (mode == MODE_CHUNK_SCAN && split.cpc > 1) ? split.cpc : 1;
  const bool multi = kp.cpc > 1;
  kp.x = static_cast<const __nv_bfloat16*>(p.x);
  kp.sx = p.sx;
  kp.ldx = p.ldx;
  kp.y = static_cast<__nv_bfloat16*>(y);
  kp.sy = p.sy;
  kp.trace = trace;
  kp.withhold_loads = withhold_loads;
  kp.ss_in = (norm && mode == MODE_SCAN) ? norm->ss_in : nullptr;
  kp.ss_out = (norm && mode == MODE_SCAN) ? norm->ss_out : nullptr;
  kp.sss = norm ? norm->batch_stride : 0;
  kp.norm_eps = norm ? norm->eps : 0.f;
  kp.inv_feat = 1.0f / (float)(p.H * P);
  // the shared-memory opt-in once per device (not stream work; keeps launches
  // free of other API calls, e.g. inside a CUDA graph capture)
  static std::atomic<unsigned long long> attr_set{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set.load() & bit)) {
    const void* fns[5] = {(const void*)k_ssd_fused<false, false>, (const void*)k_ssd_fused<true, false>,
                          (const void*)k_ssd_fused<false, true>, (const void*)k_ssd_fused<true, true>,
                          (const void*)k_ssd_fused<false, false, true>};
    for (int i = 0; i < 5 && e == cudaSuccess; ++i)
      e = cudaFuncSetAttribute(fns[i], cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit);
  }
  const int64_t ctas = mode == fused::MODE_SCAN ? p.B * p.H
                                                : kp.whole + (p.B * p.H - kp.seq0) * ceil_div(p.nc, (int64_t)kp.cpc);
  if (kp.whole < 0 || kp.whole > kp.seq0 || kp.seq0 > p.B * p.H || ctas <= 0 || ctas >= (1ll << 31))
    return cudaErrorInvalidValue;
  // the dt-scaled input whenever dt is read here (the whole scan, and the step
  // modes without a step-1 output)
  const bool xdt = p.input_dt && (mode == fused::MODE_SCAN || !lam), nrm = kp.ss_in != nullptr || kp.ss_out != nullptr;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = split.programmatic ? 1 : 0;
  if (multi) {
    if (xdt || nrm || kp.whole != 0) return cudaErrorInvalidValue;
    return cudaLaunchKernelEx(&cfg, k_ssd_fused<false, false, true>, kp, mx, mb, mc, my);
  }
  if (xdt && nrm) return cudaLaunchKernelEx(&cfg, k_ssd_fused<true, true>, kp, mx, mb, mc, my);
  if (xdt) return cudaLaunchKernelEx(&cfg, k_ssd_fused<true, false>, kp, mx, mb, mc, my);
  if (nrm) return cudaLaunchKernelEx(&cfg, k_ssd_fused<false, true>, kp, mx, mb, mc, my);
  return cudaLaunchKernelEx(&cfg, k_ssd_fused<false, false>, kp, mx, mb, mc, my);
}

}  // namespace ssd
