// Allocation-free variant of the step-by-step scan (ssd_scan_fwd_noalloc).
//
// Some callers cannot allocate device memory at the point where they run the
// scan: code recorded into a CUDA graph while a capture is open (cudaMalloc
// is not a stream operation and is refused during capture), engines and
// plugin hosts that plan all device memory ahead and hand a kernel library
// only the tensors it reads and writes, and runtimes that fix their memory
// budget at start-up.  For them the step-by-step path takes its scratch (the
// log-decay sums and the per-chunk states) from a buffer compiled into the
// library instead of a caller-provided workspace.
//
// The buffer is a file-scope __device__ array: every GPU that loads libssd
// holds its kScratchBytes until the process exits.  In host code the array's
// name is only a host-side stand-in, so its device address is looked up with
// cudaGetSymbolAddress, once per device, with that device current.
#include <mutex>

#include "ssd_common.cuh"

namespace ssd {
namespace noalloc {

constexpr size_t kScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

static std::mutex g_mu;
static void* g_addr[kMaxDevices];

// Device address of g_scratch on the current device (looked up on first use).
static cudaError_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace noalloc
}  // namespace ssd

// The entry point.  libssd.cu compiles this file in the same translation unit
// as ssd_api.cu, whose validation and launch helpers it reuses unchanged.
extern "C" ssd_status ssd_scan_fwd_noalloc(const ssd_dims* d, const void* x, const float* dt, const float* A,
                                           const void* Bm, const void* Cm, const float* D, const float* init_state,
                                           void* y, float* final_state, void* stream) {
  using namespace ssd;
  ssd_status s = validate_dims(d);
  if (s != SSD_OK) return s;
  if (d->flags & SSD_FLAG_INPUT_DT) return SSD_ERR_UNSUPPORTED;  // the step-by-step path
  s = validate_scan_args(d, x, dt, A, Bm, Cm, D, init_state, y, final_state);
  if (s != SSD_OK) return s;
  Problem p = make_problem(d);
  if (unfused_ws_bytes(p) > noalloc::kScratchBytes) {
    fprintf(stderr, "libssd: ssd_scan_fwd_noalloc needs %zu scratch bytes, the built-in buffer holds %zu\n",
            unfused_ws_bytes(p), noalloc::kScratchBytes);
    return SSD_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  const cudaError_t e = noalloc::scratch_address(&scratch);
  if (e != cudaSuccess) return cuda_status(e);
  p.x = x; p.dt = dt; p.A = A; p.Bm = Bm; p.Cm = Cm; p.D = D; p.y = y;
  return run_unfused(p, init_state, final_state, static_cast<char*>(scratch), static_cast<cudaStream_t>(stream));
}
