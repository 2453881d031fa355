// Fused tensor-core kernel of the chunked SSD scan for two heads of a group
// per CTA (sm_100a): all four steps of "分块推理：解锁循环模型并行计算，实现长序列高效处理"
// §2.1-§2.2 in one pass, the inter-chunk state carried on chip.
//
// Heads h0 and h0+1 of one group read the same B and C, so one CTA loads the
// B/C tiles once, forms S = C B^T once, and runs the two state products as
// single N = 128 tensor-core instructions (the heads side by side along N).
// Per 128-token sub-chunk k (a Q = 256 chunk is two of them: the page's
// intra/inter split applied once more inside the chunk, exact by its §2.3),
// with lam the in-sub-chunk cumulative sum of dt*A of each head:
//   S          = C_k B_k^T                                (128x128x128, shared)
//   P_h        = S (.) exp(lam_t - lam_s) [s <= t]        (per head, bf16 in TMEM)
//   y_inter    = C_k [s_a | s_b](k-1)                     (N = 128)
//   b_intra    = B_k^T [X'_a | X'_b],  X'_h = diag(exp(lam_end - lam_s)) X_h   (N = 128)
//   y_intra_h  = P_h X_h                                  (A operand from TMEM)
//   y_t        = y_intra + exp(lam_t) y_inter + D x_t      (fp32)
//   s_h(k)     = exp(lam_end) s_h(k-1) + b_intra_h         (fp32, in TMEM: the b_intra
//                                                           MMA accumulates onto the scaled state)
// (with the dt-scaled input every column s of P and row s of X' also carries dt_s).
//
// Warp roles (384 threads): lane 0 of warp 0 issues the TMA loads -- x (two
// stages, both heads), B and C (one buffer) -- and L2 prefetches, and never
// blocks; lane 1 of warp 0 stores finished y tiles (the two lanes diverge and
// each runs while the other waits); warp 1
// owns TMEM and issues the MMAs in the order S, y_inter, b_intra, y_intra;
// warps 2-3 load dt, scan lam and write X'; warps 4-7 / 8-11 are the warps of
// head a / b (warp w owns TMEM lane quarter w % 4, one thread per row): they
// turn S into that head's P, then update its state and finish its y.  The two
// heads' masks thus run side by side, two warps per SM sub-partition.  The x
// tile of a head is also where its y tile is staged for the TMA store: each
// thread reads its own x row and overwrites it with its y row; the store lane
// stores the tile once all 128 rows are staged and, once the store has read
// both heads' tiles, frees the x stage for the next load.  No head warp waits
// for a store, and no load waits behind one.
//
// TMEM (512 columns): two 128-column regions SP[0], SP[1] take turns -- S(k)
// goes to SP[k&1], P(k) to SP[1-(k&1)], y_intra(k) back to SP[k&1] -- so S of
// the next sub-chunk (issued once y_intra(k), the reader of P(k), completed)
// runs while this one's outputs are being read; y_inter
// has 128 columns, and the running fp32 state of both heads lives in the last
// 128 (after b_intra(k) it holds s(k); the head warps read it, publish its
// bf16 copy for y_inter(k+1), and write exp(lam_end(k+1)) s(k) back for the
// b_intra(k+1) MMA to accumulate onto).
//
// Work split (csrc/ssd_split.cuh): with a workspace and at least as many
// (batch, head pair) sequences as SMs, one persistent CTA per SM runs
// (segment, sequence) items round-robin, numbered segment-major; a segment
// after the first starts from the end state its predecessor published to the
// sequence's workspace slot (the page's §2.2 recursion: the carry is b(c-1)
// of the next chunk).  Without a workspace every CTA runs whole sequences.
//
// Every wait is bounded (about one second); a wait that gives up raises the
// device status word, and every role then runs its loop to the end without
// issuing further asynchronous work (TMA, MMA), still arriving once per phase
// on every barrier it arrives on, so no barrier phase is left half-counted and
// no copy is in flight when the CTA exits.
#include "ssd_common.cuh"
#include "ssd_split.cuh"
#include "tma.cuh"
#include "umma.cuh"

namespace ssd {
namespace pair {

using namespace umma;
using split::Rounds;
using split::ld_acquire;
using split::st_release;

constexpr int T = 128;   // tokens per sub-chunk
constexpr int P = 64;    // head dim
constexpr int NS = 128;  // state dim
constexpr int THREADS = 384;
constexpr uint32_t TILE = 16384;  // [128 rows][64 bf16], 128B-swizzled

constexpr uint32_t OFF_B = 0;                    // B tile: n-blocks 0-63, 64-127
constexpr uint32_t OFF_C = 2 * TILE;             // C tile
constexpr uint32_t OFF_X = 4 * TILE;             // x: [stage 2][head 2] tiles (y staged in place)
constexpr uint32_t OFF_XP = 8 * TILE;            // X': [head 2] tiles (one N = 128 operand)
constexpr uint32_t OFF_ST = 10 * TILE;           // bf16 state: [head 2] tiles, MN-major [n][p]
constexpr uint32_t OFF_TAB = 12 * TILE;          // float tables [slot 4][head 2][lam, ec, dts][128]
constexpr uint32_t TAB_BYTES = 4 * 2 * 3 * T * 4;
constexpr uint32_t OFF_WTOT = OFF_TAB + TAB_BYTES;  // scan partials [head 2][warp 2]
constexpr uint32_t OFF_BAR = OFF_WTOT + 64;
constexpr uint32_t NBAR = 22;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 64 + 1024;  // + alignment slack
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_SP = 0, TM_YI = 256, TM_BI = 384;  // SP[i] at 128*i

enum {
  BCFULL = 0,     // B/C tiles landed (tx)
  SFULL = 1,      // S complete
  BIFULL = 2,     // y_inter and b_intra complete (B/C, X' and the bf16 state free; s(k) readable)
  YFULL = 3,      // y_intra of both heads complete
  PFULL = 4,      // P of both heads written (256 head threads)
  XPFULL = 5,     // X' written (64 aux threads)
  BIREADY = 6,    // the state region holds exp(lam_end(k)) s(k-1) for b_intra(k) (256)
  STATEFULL = 7,  // bf16 state published (256)
  YEMPTY = 8,     // y_inter read (256)
  XFULL0 = 9,     // [stage] x tiles landed (tx)
  YSTAGED0 = 11,  // [stage][head] 128 y rows of the head staged in its x tile (128); one barrier per
                  // stage, so the head warps cannot complete a second phase before the store lane has
                  // seen the first (the stage is reloaded only after its y was stored)
  LAMRDY0 = 15,   // [slot 4] tables written (64 aux threads)
  DRAIN = 19,
  XEMPTY0 = 20    // [stage] both y tiles stored from the stage and read (store lane, 1)
};
constexpr int AUX = 64, HEADT = 128, EPIT = 256;
constexpr int W_TMA = 0, W_MMA = 1;

struct Params {
  int64_t L;
  int H, G, nsub;   // nsub = ceil(L / T)
  int64_t npairs;   // B * H / 2: the sequences of the schedule
  int nseg;         // segments per sequence
  int nctas;
  const float* dt;
  int64_t sdt, lddt;
  const float* A;
  const float* D;
  const float* init;
  float* final_state;
  const __nv_bfloat16* x;  // only its layout is used here (TMA maps); kept for completeness
  float* carry;            // [npairs][2][NS][P] end state of the last finished segment, or NULL
  int* carry_flag;         // [npairs] segments whose end state is published, zeroed before the launch
  int withhold;            // self-test of the bounded waits: 1 = no TMA loads, 2 = no carries published
};

struct Ctl {
  uint64_t* bar;
  volatile int* abort;
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
          give_up();
          return false;
        }
      }
    }
  }
  __device__ void give_up() const {
    *abort = 1;
    atomicExch(&g_device_status, 2);
  }
};

__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n)); }

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
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

// Packed fp32x2 arithmetic (sm_100): each lane rounded like the scalar op.
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

template <bool XDT>
__global__ void __launch_bounds__(THREADS, 1)
    k_ssd_pair(Params p, const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_b,
               const __grid_constant__ CUtensorMap map_c, const __grid_constant__ CUtensorMap map_y) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(sm);
  float* tabs = reinterpret_cast<float*>(sm + OFF_TAB);
  float* wtot = reinterpret_cast<float*>(sm + OFF_WTOT);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(sm + OFF_MISC + 4);
  Ctl ctl{bar, abort_flag};
  // table of (slot, head, kind): kind 0 = lam (log2 units), 1 = decay to the end
  // of the column's 32-block (times dt_s with the dt-scaled input), 2 = dt_s
  auto tab = [&](int slot, int h, int kind) { return tabs + ((slot * 2 + h) * 3 + kind) * T; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hpp = p.H / 2;  // head pairs per batch
  Rounds rg;
  rg.init(p.npairs, p.nsub, p.nseg, p.nctas, blockIdx.x);
  const int64_t K = rg.count();

  if (warp == W_MMA) tmem_alloc(tmem_slot, TMEM_COLS);
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(&bar[BCFULL], 1);
    mbar_init(&bar[SFULL], 1);
    mbar_init(&bar[BIFULL], 1);
    mbar_init(&bar[YFULL], 1);
    mbar_init(&bar[PFULL], EPIT);
    mbar_init(&bar[XPFULL], AUX);
    mbar_init(&bar[BIREADY], EPIT);
    mbar_init(&bar[STATEFULL], EPIT);
    mbar_init(&bar[YEMPTY], EPIT);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar[XFULL0 + i], 1);
      mbar_init(&bar[XEMPTY0 + i], 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&bar[YSTAGED0 + i], HEADT);
    for (int i = 0; i < 4; ++i) mbar_init(&bar[LAMRDY0 + i], AUX);
    mbar_init(&bar[DRAIN], 1);
    fence_mbar_init();
    prefetch_tmap(&map_x);
    prefetch_tmap(&map_b);
    prefetch_tmap(&map_c);
    prefetch_tmap(&map_y);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto coords = [&](int64_t k, int& b, int& h0, int& g, int& t0) {
    int64_t u;
    int j, r;
    bool f, l, ci, co;
    rg.at(k, u, j, r, f, l, ci, co);
    b = (int)(u / hpp);
    h0 = (int)(u % hpp) * 2;
    g = h0 / (p.H / p.G);
    t0 = j * T;
  };

  if (warp == W_TMA) {
    // ------------------------------------------------------------ TMA producer
    // Two queues polled in turn: B/C of sub-chunk kb (one buffer, free once
    // y_inter and b_intra of kb-1 completed) and x of sub-chunk kx (two stages,
    // free once the store warp has stored both heads' y tiles of kx-2).
    if (lane == 0) {
      constexpr int kPrefetch = 3;
      auto prefetch = [&](int64_t k) {
        if (k >= K) return;
        int b, h0, g, t0;
        coords(k, b, h0, g, t0);
        tma_prefetch_4d(&map_x, 0, h0, t0, b);
        tma_prefetch_4d(&map_x, 0, h0 + 1, t0, b);
        tma_prefetch_4d(&map_b, 0, g, t0, b);
        tma_prefetch_4d(&map_b, 64, g, t0, b);
        tma_prefetch_4d(&map_c, 0, g, t0, b);
        tma_prefetch_4d(&map_c, 64, g, t0, b);
      };
      for (int64_t k = 0; k < kPrefetch; ++k) prefetch(k);
      const bool loads = p.withhold != 1;
      int64_t kb = 0, kx = 0, pf = kPrefetch;
      uint32_t idle = 0;
      uint64_t t_last = globaltimer_ns();
      while ((kb < K || kx < K) && !*abort_flag) {
        bool progress = false;
        if (kb < K && (kb < 1 || mbar_test_wait(&bar[BIFULL], (kb - 1) & 1))) {
          int b, h0, g, t0;
          coords(kb, b, h0, g, t0);
          if (loads) {
            mbar_arrive_expect_tx(&bar[BCFULL], 4 * TILE);
            tma_load_4d(sm + OFF_B, &map_b, &bar[BCFULL], 0, g, t0, b);
            tma_load_4d(sm + OFF_B + TILE, &map_b, &bar[BCFULL], 64, g, t0, b);
            tma_load_4d(sm + OFF_C, &map_c, &bar[BCFULL], 0, g, t0, b);
            tma_load_4d(sm + OFF_C + TILE, &map_c, &bar[BCFULL], 64, g, t0, b);
          }
          ++kb;
          if (pf < kb + kPrefetch) prefetch(pf++);
          progress = true;
        }
        if (kx < K && kx <= kb + 1 &&
            (kx < 2 || mbar_test_wait(&bar[XEMPTY0 + (kx & 1)], (uint32_t)(((kx - 2) >> 1) & 1)))) {
          int b, h0, g, t0;
          coords(kx, b, h0, g, t0);
          const int st = (int)(kx & 1);
          uint8_t* dst = sm + OFF_X + st * 2 * TILE;
          if (loads) {
            mbar_arrive_expect_tx(&bar[XFULL0 + st], 2 * TILE);
            tma_load_4d(dst, &map_x, &bar[XFULL0 + st], 0, h0, t0, b);
            tma_load_4d(dst + TILE, &map_x, &bar[XFULL0 + st], 0, h0 + 1, t0, b);
          }
          ++kx;
          progress = true;
        }
        if (progress) {
          idle = 0;
        } else if ((++idle & 63) == 0) {
          const uint64_t now = globaltimer_ns();
          if (idle == 64) t_last = now;
          if (now - t_last > 1000000000ull) {
            ctl.give_up();
            break;
          }
        } else {
          __nanosleep(32);
        }
      }
      // every load issued must land before the CTA may exit (bounded: valid
      // tiles land unless the device is wedged)
      if (loads) {
        const uint64_t t0 = globaltimer_ns();
        if (kb > 0)
          while (!mbar_try_wait(&bar[BCFULL], (kb - 1) & 1) && globaltimer_ns() - t0 < 1000000000ull) {
          }
        for (int64_t k = (kx > 2 ? kx - 2 : 0); k < kx; ++k)
          while (!mbar_try_wait(&bar[XFULL0 + (k & 1)], (k >> 1) & 1) && globaltimer_ns() - t0 < 1000000000ull) {
          }
      }
    }
    if (lane == 1) {
      // ---------------------------------------------------------- y stores
      // head a then head b of each sub-chunk once its 128 rows are staged;
      // then wait until both stores have read the stage and free it for x(k+2)
      for (int64_t k = 0; k < K; ++k) {
        int b, h0, g, t0;
        coords(k, b, h0, g, t0);
        const int st = (int)(k & 1);
#pragma unroll 1
        for (int hy = 0; hy < 2; ++hy) {
          const bool ok = ctl.wait(YSTAGED0 + 2 * st + hy, (uint32_t)((k >> 1) & 1));
          if (ok) {
            tma_store_4d(&map_y, sm + OFF_X + st * 2 * TILE + hy * TILE, 0, h0 + hy, t0, b);
            tma_store_commit();
          }
        }
        tma_store_wait_read0();
        mbar_arrive(&bar[XEMPTY0 + st]);
      }
      tma_store_wait0();  // the y tiles are in global memory before the CTA exits
    }
  } else if (warp == W_MMA) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16(128, 128, false, false);   // C (K-major) x B^T (K-major)
      const uint32_t idYI = idesc_bf16(128, 128, false, true);   // C x [s_a|s_b] (MN-major)
      const uint32_t idBI = idesc_bf16(128, 128, true, true);    // B^T (MN-major) x [X'_a|X'_b] (MN-major)
      const uint32_t idY = idesc_bf16(128, 64, false, true);     // P (TMEM) x X (MN-major)
      const uint64_t dC = smem_desc(sbase + OFF_C, 16, 1024);
      const uint64_t dBk = smem_desc(sbase + OFF_B, 16, 1024);
      const uint64_t dBmn = smem_desc(sbase + OFF_B, TILE, 1024);
      const uint64_t dXp = smem_desc(sbase + OFF_XP, TILE, 1024);
      const uint64_t dSt = smem_desc(sbase + OFF_ST, TILE, 1024);
      const uint64_t dX = smem_desc(sbase + OFF_X, TILE, 1024);
      bool ok = true;
      for (int64_t k = 0; k < K; ++k) {
        const int pi = (int)(k & 1);
        const uint32_t tS = tmem + TM_SP + 128 * pi, tP = tmem + TM_SP + 128 * (1 - pi);
        const uint32_t ph = (uint32_t)(k & 1), php = (uint32_t)((k - 1) & 1);
        // S(k) into SP[pi], over P(k-1): the y_intra(k-1) MMAs read their A
        // operand there, and MMAs into different accumulators carry no
        // read-before-write order, so S(k) waits until they have completed
        if (ok) ok = ctl.wait(BCFULL, ph);
        if (ok && k > 0) ok = ctl.wait(YFULL, php);
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t koff = (ks >> 2) * TILE + (ks & 3) * 32;
            mma_ss(tS, desc_advance(dC, koff), desc_advance(dBk, koff), idS, ks > 0);
          }
          mma_commit(&bar[SFULL]);
        }
        // y_inter(k) = C [s_a | s_b](k-1): needs the published state and y_inter(k-1) read
        if (ok) ok = ctl.wait(STATEFULL, ph);
        if (ok && k > 0) ok = ctl.wait(YEMPTY, php);
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_ss(tmem + TM_YI, desc_advance(dC, (ks >> 2) * TILE + (ks & 3) * 32), desc_advance(dSt, ks * 2048),
                   idYI, ks > 0);
        }
        // state(k) = exp(lam_end) state(k-1) + B^T [X'_a | X'_b]: needs X'(k) and the
        // scaled state written back by the head warps
        if (ok) ok = ctl.wait(XPFULL, ph);
        if (ok) ok = ctl.wait(BIREADY, ph);
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_ss(tmem + TM_BI, desc_advance(dBmn, ks * 2048), desc_advance(dXp, ks * 2048), idBI, 1);
          mma_commit(&bar[BIFULL]);  // also: B/C, X' and the bf16 state are free again
        }
        // y_intra(k) of both heads into SP[pi] (both masks have read S there)
        if (ok) ok = ctl.wait(PFULL, ph);
        if (ok) {
          tc_fence_after();
          const uint64_t xs = desc_advance(dX, (uint32_t)(k & 1) * 2 * TILE);
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
              mma_ts(tS + 64 * h, tP + 64 * h + ks * 8, desc_advance(xs, h * TILE + ks * 2048), idY, ks > 0);
          mma_commit(&bar[YFULL]);
        }
      }
      // every MMA issued must complete before TMEM is released (also on abort)
      mma_commit(&bar[DRAIN]);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&bar[DRAIN], 0) && globaltimer_ns() - t0 < 1000000000ull) {
      }
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ dt, lam, decay tables, X'
    const int a = threadIdx.x - 64;  // 0..63 (warps 2-3)
    const int aw = warp - 2;
    auto load_dt = [&](int64_t k, float (&d)[2][2], float (&Ah)[2]) {
      if (k >= K) {
        d[0][0] = d[0][1] = d[1][0] = d[1][1] = 0.f;
        return;
      }
      int64_t u;
      int j, r;
      bool f, l, ci, co;
      rg.at(k, u, j, r, f, l, ci, co);
      const int b = (int)(u / hpp), h0 = (int)(u % hpp) * 2;
      const float* dtb = p.dt + (int64_t)b * p.sdt + h0;
      const int64_t t0 = (int64_t)j * T + 2 * a;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        Ah[h] = p.A[h0 + h];
        d[h][0] = (t0 < p.L) ? dtb[t0 * p.lddt + h] : 0.f;
        d[h][1] = (t0 + 1 < p.L) ? dtb[(t0 + 1) * p.lddt + h] : 0.f;
      }
    };
    float d[2][2], Ah[2];
    load_dt(0, d, Ah);
    for (int64_t k = 0; k < K; ++k) {
      const int slot = (int)(k & 3), st = (int)(k & 1);
      float dn[2][2], An[2];
      load_dt(k + 1, dn, An);  // one sub-chunk ahead
      // inclusive scans of dt*A over the 128 tokens (two per thread), both heads
      float l0[2], l1[2], v[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        l0[h] = d[h][0] * Ah[h];
        l1[h] = d[h][1] * Ah[h];
        v[h] = l0[h] + l1[h];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const float nb = __shfl_up_sync(0xffffffffu, v[h], off);
          if (lane >= off) v[h] += nb;
        }
        if (lane == 31) wtot[h * 2 + aw] = v[h];
      }
      named_sync(1, AUX);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float pre = (aw == 1) ? wtot[h * 2] : 0.f;
        const float lam1 = v[h] + pre, lam0 = lam1 - l1[h];
        float* lj = tab(slot, h, 0);
        lj[2 * a] = lam0 * kLog2e;
        lj[2 * a + 1] = lam1 * kLog2e;
        if constexpr (XDT) {
          float* dts = tab(slot, h, 2);
          dts[2 * a] = d[h][0];
          dts[2 * a + 1] = d[h][1];
        }
      }
      named_sync(1, AUX);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float* lj = tab(slot, h, 0);
        float* ec = tab(slot, h, 1);
        const float lr = lj[(2 * a) | 31];
        float e0 = ex2(lr - lj[2 * a]), e1 = ex2(lr - lj[2 * a + 1]);
        if constexpr (XDT) {
          e0 *= d[h][0];
          e1 *= d[h][1];
        }
        ec[2 * a] = e0;
        ec[2 * a + 1] = e1;
      }
      mbar_arrive(&bar[LAMRDY0 + slot]);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        Ah[h] = An[h];
        d[h][0] = dn[h][0];
        d[h][1] = dn[h][1];
      }
      // X'(k) = diag(exp(lam_end - lam_t)) X(k), both heads, rows a and a + 64,
      // once x(k) landed and b_intra(k-1) (the last reader of X') completed
      bool ok = ctl.wait(XFULL0 + st, (uint32_t)((k >> 1) & 1));
      if (ok && k > 0) ok = ctl.wait(BIFULL, (uint32_t)((k - 1) & 1));
      if (ok) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float* lj = tab(slot, h, 0);
          const float lam_end = lj[T - 1];
          const uint32_t src = sbase + OFF_X + st * 2 * TILE + h * TILE;
          const uint32_t dst = sbase + OFF_XP + h * TILE;
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const int row = a + 64 * rr;
            float w = ex2(lam_end - lj[row]);
            if constexpr (XDT) w *= tab(slot, h, 2)[row];
            const float2 w2 = make_float2(w, w);
            uint4 v4[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) v4[c] = lds128(src + swz128(row, c * 8));
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint32_t* u = reinterpret_cast<uint32_t*>(&v4[c]);
#pragma unroll
              for (int i = 0; i < 4; ++i) {  // fp32 product, one rounding
                const float2 f = mul2(bf2_to_f2(u[i]), w2);
                u[i] = pack_bf16(f.x, f.y);
              }
              sts128(dst + swz128(row, c * 8), v4[c]);
            }
          }
        }
        fence_async_smem();
      }
      mbar_arrive(&bar[XPFULL]);
      named_sync(1, AUX);  // wtot reuse
    }
  } else {
    // ------------------------------------------------------------ the warps of head hl
    const int hl = (warp - 4) >> 2;  // 0: warps 4-7, 1: warps 8-11
    const int q = warp & 3;          // TMEM lane quarter
    const int r = q * 32 + lane;     // S / P / y row t and state row n
    const int et = threadIdx.x - 128;  // 0..255 over both heads
    const uint32_t lq = (uint32_t)(q * 32) << 16;
    const uint32_t sSt = sbase + OFF_ST + hl * TILE;
    const uint32_t tSt = tmem + lq + TM_BI + 64 * hl;  // this head's fp32 state, row r
    // Columns 32c..32c+31 of the state row: the bf16 copy into the MN-major
    // operand tile of y_inter, and dec times the values back into TMEM.
    auto publish_half = [&](int c, const uint32_t* v) {
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        uint4 w;
        w.x = pack_bf16(__uint_as_float(v[8 * c8 + 0]), __uint_as_float(v[8 * c8 + 1]));
        w.y = pack_bf16(__uint_as_float(v[8 * c8 + 2]), __uint_as_float(v[8 * c8 + 3]));
        w.z = pack_bf16(__uint_as_float(v[8 * c8 + 4]), __uint_as_float(v[8 * c8 + 5]));
        w.w = pack_bf16(__uint_as_float(v[8 * c8 + 6]), __uint_as_float(v[8 * c8 + 7]));
        sts128(sSt + swz128(r, 32 * c + 8 * c8), w);
      }
    };
    auto scale_back = [&](int c, uint32_t* v, float dec) {
      const float2 dec2 = make_float2(dec, dec);
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float2 o = mul2(dec2, make_float2(__uint_as_float(v[i]), __uint_as_float(v[i + 1])));
        v[i] = __float_as_uint(o.x);
        v[i + 1] = __float_as_uint(o.y);
      }
      tmem_st32(tSt + 32 * c, v);
    };
    float Dh = 0.f;
    int64_t u = -1;
    int b = 0, h = 0;
    for (int64_t k = 0; k < K; ++k) {
      int j, seg;
      bool first, last, carry_in, carry_out;
      rg.at(k, u, j, seg, first, last, carry_in, carry_out);
      if (first) {
        // a new piece: its initial state (given, carried or zero) is published
        // for y_inter(k) and written, times exp(lam_end(k)), for b_intra(k)
        b = (int)(u / hpp);
        h = (int)(u % hpp) * 2 + hl;
        Dh = p.D ? p.D[h] : 0.f;
        const float* src = nullptr;
        if (carry_in) {
          // segment seg - 1 of this sequence (an item at least one round
          // earlier, normally finished) publishes its end state; wait for it
          const int* flag = p.carry_flag + u;
          if (ld_acquire(flag) < seg) {
            const uint64_t t0 = globaltimer_ns();
            bool done = false;
            while (!done && !*abort_flag) {
              __nanosleep(256);
              done = ld_acquire(flag) >= seg;
              if (!done && globaltimer_ns() - t0 > 2000000000ull) {
                ctl.give_up();
                break;
              }
            }
          }
          src = p.carry + (u * 2 + hl) * NS * P;
        } else if (p.init) {
          src = p.init + ((int64_t)b * p.H + h) * NS * P;
        }
        if (src && *abort_flag) src = nullptr;
        ctl.wait(LAMRDY0 + (int)(k & 3), (uint32_t)((k >> 2) & 1));
        const float dec = ex2(tab((int)(k & 3), hl, 0)[T - 1]);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t v[32];
          if (src) {
            const float4* s4 = reinterpret_cast<const float4*>(src + (int64_t)r * P + 32 * c);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 f = s4[i];
              v[4 * i] = __float_as_uint(f.x);
              v[4 * i + 1] = __float_as_uint(f.y);
              v[4 * i + 2] = __float_as_uint(f.z);
              v[4 * i + 3] = __float_as_uint(f.w);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0u;
          }
          publish_half(c, v);
          scale_back(c, v, dec);
        }
        fence_async_smem();
        mbar_arrive(&bar[STATEFULL]);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar[BIREADY]);
      }
      const int slot = (int)(k & 3), pi = (int)(k & 1), st = (int)(k & 1);
      const float* lj = tab(slot, hl, 0);
      // ---- P = S (.) L of this head into SP[1-pi], columns 64 hl .. +63
      {
        bool ok = ctl.wait(LAMRDY0 + slot, (uint32_t)((k >> 2) & 1));
        if (ok) ok = ctl.wait(SFULL, (uint32_t)(k & 1));
        (void)ok;
        tc_fence_after();
        const uint32_t tS = tmem + lq + TM_SP + 128 * pi, tP = tmem + lq + TM_SP + 128 * (1 - pi) + 64 * hl;
        const float lam_t = lj[r];
        const float* ec = tab(slot, hl, 1);
        auto make_block = [&](int kb, const uint32_t* rv, uint32_t* pk) {
          if (kb < q) {
            // below the diagonal block: exp(lam_t - lam_s) = 2^(lt - l_end(kb)) * ec[s]
            const float4* ec4 = reinterpret_cast<const float4*>(ec);
            const float rowf = ex2(lam_t - lj[32 * kb + 31]);
            const float2 rf2 = make_float2(rowf, rowf);
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              const float4 c = ec4[8 * kb + v];
              const float2 a0 = mul2(mul2(make_float2(__uint_as_float(rv[4 * v]), __uint_as_float(rv[4 * v + 1])),
                                          make_float2(c.x, c.y)),
                                     rf2);
              const float2 a1 = mul2(mul2(make_float2(__uint_as_float(rv[4 * v + 2]), __uint_as_float(rv[4 * v + 3])),
                                          make_float2(c.z, c.w)),
                                     rf2);
              pk[2 * v] = pack_bf16(a0.x, a0.y);
              pk[2 * v + 1] = pack_bf16(a1.x, a1.y);
            }
          } else if (kb == q) {
            // diagonal block: direct decays, clamped at 0 above the diagonal and then zeroed
            const float4* lj4 = reinterpret_cast<const float4*>(lj);
            const int rl = r - 32 * kb;
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              const float4 l = lj4[8 * kb + v];
              float e0 = ex2(fminf(lam_t - l.x, 0.f)), e1 = ex2(fminf(lam_t - l.y, 0.f));
              float e2 = ex2(fminf(lam_t - l.z, 0.f)), e3 = ex2(fminf(lam_t - l.w, 0.f));
              if constexpr (XDT) {
                const float4 fx = reinterpret_cast<const float4*>(tab(slot, hl, 2))[8 * kb + v];
                e0 *= fx.x;
                e1 *= fx.y;
                e2 *= fx.z;
                e3 *= fx.w;
              }
              const float f0 = (4 * v + 0 <= rl) ? __uint_as_float(rv[4 * v + 0]) * e0 : 0.f;
              const float f1 = (4 * v + 1 <= rl) ? __uint_as_float(rv[4 * v + 1]) * e1 : 0.f;
              const float f2 = (4 * v + 2 <= rl) ? __uint_as_float(rv[4 * v + 2]) * e2 : 0.f;
              const float f3 = (4 * v + 3 <= rl) ? __uint_as_float(rv[4 * v + 3]) * e3 : 0.f;
              pk[2 * v] = pack_bf16(f0, f1);
              pk[2 * v + 1] = pack_bf16(f2, f3);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = 0u;
          }
        };
        // one 32-column block per TMEM round trip (as in the one-head kernel)
#pragma unroll 1
        for (int kb = 0; kb < 4; ++kb) {
          uint32_t r0[32], pk[16];
          // warp-uniform: only blocks on or below the diagonal block are read
          if (kb <= q) {
            tmem_ld32(tS + 32 * kb, r0);
            tmem_wait_ld();
          }
          make_block(kb, r0, pk);
          tmem_st16(tP + 16 * kb, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar[PFULL]);
      }
      // ---- state: the MMA left s(k) = exp(lam_end) s(k-1) + b_intra(k) in TMEM
      bool ok = ctl.wait(BIFULL, (uint32_t)(k & 1));
      tc_fence_after();
      if (!last) {
        // publish bf16 s(k) for y_inter(k+1) (y_inter(k) has completed: BIFULL
        // covers it) and write exp(lam_end(k+1)) s(k) back for b_intra(k+1)
        ctl.wait(LAMRDY0 + (int)((k + 1) & 3), (uint32_t)(((k + 1) >> 2) & 1));
        const float dec = ex2(tab((int)((k + 1) & 3), hl, 0)[T - 1]);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t v[32];
          tmem_ld32(tSt + 32 * c, v);
          tmem_wait_ld();
          publish_half(c, v);
          scale_back(c, v, dec);
        }
        fence_async_smem();
        mbar_arrive(&bar[STATEFULL]);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar[BIREADY]);
      } else {
        // end of a segment: the sequence's final state, or the carry of the next
        // segment (the slot was read at this segment's start)
        float* dst = nullptr;
        if (carry_out)
          dst = p.carry + (u * 2 + hl) * NS * P;
        else if (p.final_state)
          dst = p.final_state + ((int64_t)b * p.H + h) * NS * P;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t v[32];
          tmem_ld32(tSt + 32 * c, v);
          tmem_wait_ld();
          if (dst) {
            float4* d4 = reinterpret_cast<float4*>(dst + (int64_t)r * P + 32 * c);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              d4[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                  __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
          }
        }
        tc_fence_before();
        if (carry_out) {
          __threadfence();
          named_sync(2, EPIT);
          if (et == 0 && p.withhold != 2) st_release(p.carry_flag + u, seg + 1);
        }
      }
      // ---- y_t = y_intra + exp(lam_t) y_inter + D x_t, written over this head's
      // x row (each thread reads and writes only its own row); the producer
      // stores the tile once all 128 rows are staged
      if (ok) ok = ctl.wait(YFULL, (uint32_t)(k & 1));
      tc_fence_after();
      const float etl = ex2(lj[r]);
      const uint32_t xrow = sbase + OFF_X + st * 2 * TILE + hl * TILE;
      const uint32_t tY = tmem + lq + TM_SP + 128 * pi + 64 * hl, tI = tmem + lq + TM_YI + 64 * hl;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t yi[16], ye[16];
        tmem_ld16(tY + 16 * c, yi);
        tmem_ld16(tI + 16 * c, ye);
        const uint4 xa = lds128(xrow + swz128(r, 16 * c));
        const uint4 xb = lds128(xrow + swz128(r, 16 * c + 8));
        tmem_wait_ld();
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const uint4 xv = h2 ? xb : xa;
          const uint32_t* xu = reinterpret_cast<const uint32_t*>(&xv);
          uint4 ov;
          uint32_t* o = reinterpret_cast<uint32_t*>(&ov);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int k0 = h2 * 8 + 2 * i;
            float2 yo = fma2(make_float2(Dh, Dh), bf2_to_f2(xu[i]),
                             make_float2(__uint_as_float(yi[k0]), __uint_as_float(yi[k0 + 1])));
            yo = fma2(make_float2(etl, etl), make_float2(__uint_as_float(ye[k0]), __uint_as_float(ye[k0 + 1])), yo);
            o[i] = pack_bf16(yo.x, yo.y);
          }
          sts128(xrow + swz128(r, 16 * c + 8 * h2), ov);
        }
      }
      tc_fence_before();
      mbar_arrive(&bar[YEMPTY]);
      fence_async_smem();  // the y rows are visible to the store (async proxy)
      mbar_arrive(&bar[YSTAGED0 + 2 * st + hl]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
    tmem_relinquish();
  }
}

}  // namespace pair

// Two heads of one group per CTA: the head count per group must be even.
bool pair_supported(const Problem& p) {
  return p.io == SSD_BF16 && p.P == pair::P && p.N == pair::NS && p.Q % pair::T == 0 && (p.H / p.G) % 2 == 0 &&
         p.B * p.H < (1ll << 31);
}

// Segments per sequence (csrc/ssd_split.cuh), or the count a self-test set.
static int g_segments_override = 0;
void set_pair_segments(int nseg) { g_segments_override = nseg > 0 ? nseg : 0; }
static int pair_segments(const Problem& p) {
  const int nsub = (int)ceil_div(p.L, (int64_t)pair::T);
  if (g_segments_override > 0) return (nsub % g_segments_override == 0) ? g_segments_override : 1;
  return split::segments(p.B * p.H / 2, nsub, split::sm_count());
}

// CTAs of the segmented schedule: one per SM, never more than the items.
int pair_split_ctas(const Problem& p) {
  const int64_t items = p.B * p.H / 2 * pair_segments(p);
  const int n = split::sm_count();
  return (int)(items < n ? items : n);
}

// Workspace of the segmented schedule: one carry slot [2][N][P] f32 per head
// pair and their flags, or 0 when the sequences run whole.
size_t pair_workspace_bytes(const Problem& p) {
  if (!pair_supported(p)) return 0;
  return split::workspace_bytes(p.B * p.H / 2, pair_segments(p), (size_t)2 * pair::NS * pair::P);
}

// withhold: 0 normal; 1 issue no TMA loads (self-test of the bounded waits);
// 2 publish no carries (self-test of the carry wait; needs a split schedule).
cudaError_t launch_pair(const Problem& p, const float* init, float* final_state, void* workspace,
                        size_t workspace_bytes, cudaStream_t st, int withhold) {
  using namespace pair;
  if (!p.x || !p.Bm || !p.Cm || !p.dt || !p.A || !p.y) return cudaErrorInvalidValue;
  CUtensorMap mx, mb, mc, my;
  const uint32_t box[4] = {64, 1, (uint32_t)T, 1};
  const uint64_t dx[4] = {(uint64_t)P, (uint64_t)p.H, (uint64_t)p.L, (uint64_t)p.B};
  const uint64_t sx[3] = {(uint64_t)P * 2, (uint64_t)p.ldx * 2, (uint64_t)p.sx * 2};
  const uint64_t sy[3] = {(uint64_t)P * 2, (uint64_t)p.ldy * 2, (uint64_t)p.sy * 2};
  const uint64_t dbc[4] = {(uint64_t)NS, (uint64_t)p.G, (uint64_t)p.L, (uint64_t)p.B};
  const uint64_t sbc[3] = {(uint64_t)NS * 2, (uint64_t)p.ldbc * 2, (uint64_t)p.sbc * 2};
  if (!tma::encode_bf16_4d_cached(&mx, p.x, dx, sx, box) || !tma::encode_bf16_4d_cached(&mb, p.Bm, dbc, sbc, box) ||
      !tma::encode_bf16_4d_cached(&mc, p.Cm, dbc, sbc, box) || !tma::encode_bf16_4d_cached(&my, p.y, dx, sy, box))
    return cudaErrorInvalidValue;
  Params kp;
  kp.L = p.L;
  kp.H = (int)p.H;
  kp.G = (int)p.G;
  kp.nsub = (int)ceil_div(p.L, T);
  kp.npairs = p.B * p.H / 2;
  kp.dt = p.dt;
  kp.sdt = p.sdt;
  kp.lddt = p.lddt;
  kp.A = p.A;
  kp.D = p.D;
  kp.init = init;
  kp.final_state = final_state;
  kp.x = static_cast<const __nv_bfloat16*>(p.x);
  kp.withhold = withhold;
  const size_t need = pair_workspace_bytes(p);
  if (need > 0 && workspace && workspace_bytes >= need) {
    kp.nseg = pair_segments(p);
    kp.nctas = pair_split_ctas(p);
    kp.carry = static_cast<float*>(workspace);
    kp.carry_flag = reinterpret_cast<int*>(static_cast<char*>(workspace) +
                                           (size_t)kp.npairs * 2 * NS * P * sizeof(float));
    cudaError_t e = cudaMemsetAsync(kp.carry_flag, 0, (size_t)kp.npairs * sizeof(int), st);
    if (e != cudaSuccess) return e;
  } else {
    kp.nseg = 1;                // whole sequences, one CTA each
    kp.nctas = (int)kp.npairs;
    kp.carry = nullptr;
    kp.carry_flag = nullptr;
  }
  // the shared-memory opt-in once per device (keeps later launches free of
  // other API calls, e.g. inside a CUDA graph capture)
  static std::atomic<unsigned long long> attr_set{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set.load() & bit)) {
    e = cudaFuncSetAttribute(k_ssd_pair<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_ssd_pair<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit);
  }
  if (p.input_dt)
    k_ssd_pair<true><<<(unsigned)kp.nctas, THREADS, SMEM_BYTES, st>>>(kp, mx, mb, mc, my);
  else
    k_ssd_pair<false><<<(unsigned)kp.nctas, THREADS, SMEM_BYTES, st>>>(kp, mx, mb, mc, my);
  return cudaGetLastError();
}

}  // namespace ssd
