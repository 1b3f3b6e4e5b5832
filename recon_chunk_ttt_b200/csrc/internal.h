// Internal host-side interface between the C-ABI layer (ttt_api.cu) and the
// kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>
#include <unordered_map>

namespace ttt {

// Fast-weight forms (ttt_config.mlp).
constexpr int kMlpSwiGLU = 0;
constexpr int kMlpLinear = 1;

// Problem description after validation.
struct Problem {
  int mlp;    // kMlpSwiGLU or kMlpLinear (then hid == d and W1 is the d x d W)
  int H, d, hid;
  int64_t n;  // tokens (update) or queries (apply)
  int renorm;
  int ns_steps;  // Newton-Schulz steps on the gradient (0: off)
};

// Split-K plan of the token reduction: S contiguous token ranges of `chunk`
// tokens (the last one shorter).  A function of (n, shape) only, so results
// are bitwise reproducible.
struct SplitPlan {
  int S;
  int64_t chunk;
};

// ---- fp32 CUDA-core check mode -------------------------------------------
SplitPlan f32_split_plan(const Problem& p);
size_t f32_workspace_bytes(const Problem& p);
// With partial_out != nullptr the update stops after the token reduction and
// writes the fixed-order sum of its splits there (layout of one split, below)
// instead of updating the weights.
cudaError_t f32_update(const Problem& p, const float* W1, const float* W2, const float* W3,
                       const float* K, const float* V, const float* eta, float* W1o, float* W2o,
                       float* W3o, __nv_bfloat16_raw* shadow, void* ws, cudaStream_t st,
                       float* partial_out = nullptr);
cudaError_t f32_apply(const Problem& p, const float* W1, const float* W2, const float* W3,
                      const float* Q, float* O, cudaStream_t st);

// ---- shared: reduce split-K partials + renormalise -----------------------
// Partials layout: [S][H][3][hid*d] floats; block 0 = P1 (G1, [hid][d]),
// block 1 = P3 (G3, [hid][d]), block 2 = P2 (-G2, [d][hid]).
// Writes W_out = renorm(W - G) in fp32 and, if shadow != nullptr, bf16.
// `scratch` holds H*(2*hid+d)*2 doubles (Frobenius mode only).
cudaError_t reduce_renorm(const Problem& p, int S, const float* partials, const float* W1,
                          const float* W2, const float* W3, float* W1o, float* W2o, float* W3o,
                          __nv_bfloat16_raw* shadow, float* scratch, cudaStream_t st);
// ---- optional Newton-Schulz orthonormalisation (kernels_ns.cu) ------------
// Workspace it needs beyond the update's own (0 when ns_steps == 0).
size_t ns_workspace_bytes(const Problem& p);
// With ns_steps > 0 and n > 0: Delta = NewtonSchulz(sum of the S partials) per
// head and matrix, then reduce_renorm of Delta as a single split; otherwise
// reduce_renorm of the partials as they are.
cudaError_t ns_then_renorm(const Problem& p, int S, const float* partials, void* ns_ws,
                           bool tensor_cores, const float* W1, const float* W2, const float* W3,
                           float* W1o, float* W2o, float* W3o, __nv_bfloat16_raw* shadow,
                           float* scratch, cudaStream_t st);
// out[i] = sum over s = 0..S-1 of partials[s * count + i], in that order.
cudaError_t sum_splits(int S, size_t count, const float* partials, float* out, cudaStream_t st);
// W2 and W3 may be NULL (linear fast weights: only the W1 block is written).
cudaError_t pack_shadow(int H, int d, int hid, const float* W1, const float* W2,
                        const float* W3, __nv_bfloat16_raw* shadow, cudaStream_t st);

// ---- linear fast weights f_W(k) = W k (kernels_linear.cu) ------------------
// Partials [S][H][d*d] hold P = Σ η v k^T (= -g); the update adds them.
SplitPlan linear_split_plan(const Problem& p);
size_t linear_workspace_bytes(const Problem& p);
cudaError_t linear_update(const Problem& p, bool bf16_tokens, const float* W, const void* K,
                          const void* V, const float* eta, float* Wo,
                          __nv_bfloat16_raw* shadow, void* ws, cudaStream_t st,
                          float* partial_out = nullptr);
// BF16_TC (bf16 = true) reads the bf16 shadow of W, FP32_CHECK the fp32 W.
cudaError_t linear_apply(const Problem& p, bool bf16, const float* W,
                         const __nv_bfloat16_raw* shadow, const void* Q, void* O,
                         cudaStream_t st);

// ---- bf16 tensor-core path (tcgen05) --------------------------------------
SplitPlan tc_split_plan(const Problem& p);
size_t tc_workspace_bytes(const Problem& p);
cudaError_t tc_update(const Problem& p, const float* W1, const float* W2, const float* W3,
                      const void* K, const void* V, const float* eta, float* W1o, float* W2o,
                      float* W3o, __nv_bfloat16_raw* shadow, void* ws, cudaStream_t st,
                      float* partial_out = nullptr);
cudaError_t tc_apply(const Problem& p, const __nv_bfloat16_raw* shadow, const void* Q, void* O,
                     cudaStream_t st);
// Fused update kernel (kernels_fused.cu): fp32 weights W1, W3 [H][hid][d],
// W2 [H][d][hid] in (rounded to bf16 inside); the S partial slots of the
// plan out ([S][H][3][hid*d]).  The head-major tile space is split over
// `sets` sets of hid/128 3-CTA clusters (one per group of 128 hidden units):
// evenly over the whole space (sets_per_head = 0), or, for few tiles per
// head, sets_per_head sets per head; a head's gradient arrives in at most
// `splits` pieces (slots), unused slots are zero.
struct FusedPlan {
  int sets, sets_per_head, splits;
};
FusedPlan fused_plan(const Problem& p);
cudaError_t fused_update(const Problem& p, const float* W1, const float* W2, const float* W3,
                         const void* K, const void* V, const float* eta, const FusedPlan& f,
                         float* partials, int* err, cudaStream_t st);
// Clusters of the fused update that fill one wave of the GPU.
int fused_clusters_per_wave();

// ---- gated output unit: o = RMSNorm(o') * SiLU(W_g o') per head ------------
// p.n = rows.  W_g [H][d][d] (row = output); bf16 (tc) or float (f32).
cudaError_t tc_gate(const Problem& p, const void* Wg, const void* Oin, void* Oout, float eps,
                    cudaStream_t st);
cudaError_t f32_gate(const Problem& p, const float* Wg, const float* Oin, float* Oout, float eps,
                     cudaStream_t st);

// One block whose bounded mbarrier wait runs out after limit_cycles.
cudaError_t selftest_wait_timeout(long long limit_cycles, cudaStream_t st);

// The per-device error word (defined in kernels_common.cu).
int* device_error_ptr();                       // device address, nullptr on failure
cudaError_t read_and_clear_device_error(int* value);

// Tracing (trace.cu): a scope records CUDA events around the launches it
// encloses when tracing is enabled through ttt_trace_enable().
bool trace_on();
class TraceScope {
 public:
  TraceScope(const char* name, cudaStream_t st);
  ~TraceScope();
  TraceScope(const TraceScope&) = delete;
  TraceScope& operator=(const TraceScope&) = delete;

 private:
  const char* name_;
  cudaStream_t st_;
  void* a_;
};

// Raise a kernel's dynamic shared-memory limit once per (kernel, device).
// Kernels of one signature share a pointer type, so the record is keyed by
// the kernel's address.
template <typename Kern>
cudaError_t ensure_smem_attr(Kern kernel, int smem) {
  static std::mutex mu;
  static std::unordered_map<const void*, uint64_t> done;  // bit = device
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const void* key = reinterpret_cast<const void*>(kernel);
  if (dev < 0 || dev >= 64)
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  std::lock_guard<std::mutex> lk(mu);
  uint64_t& bits = done[key];
  if (!(bits >> dev & 1)) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    bits |= 1ull << dev;
  }
  return cudaSuccess;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace ttt
