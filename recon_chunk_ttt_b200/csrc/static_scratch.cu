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
// (64 MiB).  Every GPU that loads this part of the library holds it until the
// process exits.  Its contents persist from call to call; nothing in it needs
// to start at zero because every kernel of the step writes the scratch it later
// reads.  All calls on a device share the one array, so two calls whose work
// can overlap on the GPU (different streams, or different host threads without
// ordering) race on it: serialise them.
//
// Host code cannot pass the array's name to a kernel (on the host it is only a
// stand-in symbol), so the device address is looked up once per device with
// cudaGetSymbolAddress() on the first call made while that device is current.
// That first call should happen before any stream capture begins.

#include <cuda_runtime.h>

#include <mutex>

#include "../../include/ttt.h"

namespace {

constexpr size_t kScratchBytes = TTT_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_static_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_static_scratch on the current device (looked up once).
ttt_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TTT_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
      return TTT_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
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
