// Allocation-free streaming step.
//
// Some callers cannot allocate device memory at the point where they run a
// frame: a real-time loop whose memory budget is fixed up front, code that runs
// inside a host-side allocator lock or a foreign runtime that owns the
// allocator, or an embedding that forbids cudaMalloc after start-up.  For them
// ttt_stream_step_static() runs the same streaming step as ttt_stream_step()
// but takes its workspace from a fixed device array that is part of the
// library image, so the call itself allocates nothing.
//
// The array is a file-scope static __device__ object of TTT_STATIC_SCRATCH_BYTES
// (96 MiB).  Every GPU that loads this part of the library holds it until the
// process exits.  Its contents persist from call to call; nothing in it needs
// to start at zero because every kernel of the step writes the scratch it later
// reads.  All calls on a device share the one array, so two calls whose work
// can overlap on the GPU (different streams, or different host threads without
// ordering) race on it: serialise them.
//
// Host code cannot pass the array's name to a kernel (on the host it is only a
// stand-in symbol), so the device address is looked up with
// cudaGetSymbolAddress() on the first call made while a device is current, and
// cached together with the unique id of that device's current CUDA context.
// When the context changes (after cudaDeviceReset, or when the primary context
// was released and created again, the module is loaded anew and the array may
// move) the id no longer matches and the address is looked up again.  A call
// that looks the address up should happen before any stream capture begins:
// the first call on each device, and the first call after such a reset.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/ttt.h"

namespace {

constexpr size_t kScratchBytes = TTT_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_static_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
struct CachedAddress {
  void* addr;
  unsigned long long ctx_id;
};
CachedAddress g_scratch[kMaxDevices] = {};
std::mutex g_scratch_mu;

// The driver's cuCtxGetCurrent / cuCtxGetId, found through the runtime (no
// link-time dependency on the driver library).
PFN_cuCtxGetCurrent_v4000 ctx_get_current() {
  static PFN_cuCtxGetCurrent_v4000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    return cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
                   q == cudaDriverEntryPointSuccess
               ? reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p)
               : nullptr;
  }();
  return fn;
}
PFN_cuCtxGetId_v12000 ctx_get_id() {
  static PFN_cuCtxGetId_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    return cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
                   q == cudaDriverEntryPointSuccess
               ? reinterpret_cast<PFN_cuCtxGetId_v12000>(p)
               : nullptr;
  }();
  return fn;
}

// Unique id of the calling thread's current context (0 if there is none or
// the driver cannot tell).
unsigned long long current_context_id() {
  auto get_current = ctx_get_current();
  auto get_id = ctx_get_id();
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_static_scratch in the current device's context.
ttt_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TTT_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  CachedAddress& c = g_scratch[dev];
  unsigned long long id = current_context_id();
  if (c.addr == nullptr || id == 0 || id != c.ctx_id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
      return TTT_ERR_CUDA;
    // the lookup makes the device's primary context current if it was not
    if (id == 0) id = current_context_id();
    c.addr = p;
    c.ctx_id = id;  // 0: unknown, looked up again on the next call
  }
  *out = c.addr;
  return TTT_OK;
}

}  // namespace

extern "C" ttt_status ttt_stream_step_static(const ttt_config* cfg, float* W1, float* W2,
                                             float* W3, void* shadow, const void* K,
                                             const void* V, const float* eta, int64_t n,
                                             const void* Q, int64_t m, void* O,
                                             ttt_stream_t stream) {
  if (cfg == nullptr) return TTT_ERR_INVALID_ARG;
  const size_t need = ttt_update_workspace_bytes(cfg, n);
  if (need > kScratchBytes) return TTT_ERR_WORKSPACE;  // problem larger than the fixed array
  void* ws = nullptr;
  const ttt_status s = scratch_address(&ws);
  if (s != TTT_OK) return s;
  return ttt_stream_step(cfg, W1, W2, W3, shadow, K, V, eta, n, Q, m, O, ws, kScratchBytes,
                         stream);
}
