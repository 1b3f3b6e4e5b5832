// C-ABI boundary (include/ttt.h): host-side validation, workspace planning and
// dispatch to the fp32 check-mode or the bf16 tensor-core kernels.  Nothing
// is enqueued unless every argument checks out.

#include <cuda_runtime.h>

#include "../../include/ttt.h"
#include "common.cuh"
#include "internal.h"

using ttt::Problem;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ttt_status check_cfg(const ttt_config* cfg) {
  if (cfg == nullptr) return TTT_ERR_INVALID_ARG;
  if (cfg->heads < 1 || cfg->heads > 4096) return TTT_ERR_INVALID_ARG;
  if (cfg->mlp != TTT_MLP_SWIGLU && cfg->mlp != TTT_MLP_LINEAR) return TTT_ERR_INVALID_ARG;
  if (cfg->renorm < TTT_RENORM_OFF || cfg->renorm > TTT_RENORM_FROB) return TTT_ERR_INVALID_ARG;
  if (cfg->precision != TTT_PREC_BF16_TC && cfg->precision != TTT_PREC_FP32_CHECK)
    return TTT_ERR_INVALID_ARG;
  if (cfg->ns_steps < 0 || cfg->ns_steps > TTT_MAX_NS_STEPS) return TTT_ERR_INVALID_ARG;
  if (cfg->mlp == TTT_MLP_LINEAR) {
    // f_W(k) = W k with W d x d (carried in W1): hidden must equal d, and the
    // Newton-Schulz switch belongs to the SwiGLU layer
    if (!((cfg->d == 64 || cfg->d == 256) && cfg->hidden == cfg->d) || cfg->ns_steps != 0)
      return TTT_ERR_UNSUPPORTED_SHAPE;
    return TTT_OK;
  }
  const bool ok = (cfg->d == 64 && cfg->hidden == 128) || (cfg->d == 256 && cfg->hidden == 512);
  if (!ok) return TTT_ERR_UNSUPPORTED_SHAPE;
  return TTT_OK;
}

bool is_linear(const ttt_config* cfg) { return cfg->mlp == TTT_MLP_LINEAR; }

// Workspace of the update of n tokens for a valid config.
size_t update_workspace(const ttt_config* cfg, const Problem& p) {
  if (is_linear(cfg)) return ttt::linear_workspace_bytes(p);
  return cfg->precision == TTT_PREC_FP32_CHECK ? ttt::f32_workspace_bytes(p)
                                               : ttt::tc_workspace_bytes(p);
}

Problem make_problem(const ttt_config* cfg, int64_t n) {
  Problem p;
  p.mlp = cfg->mlp;
  p.H = cfg->heads;
  p.d = cfg->d;
  p.hid = cfg->hidden;
  p.n = n;
  p.renorm = cfg->renorm;
  p.ns_steps = cfg->ns_steps;
  return p;
}

// Token counts are limited so that every index fits the kernels' int64
// arithmetic and the tensor-map coordinates (int32).
constexpr int64_t kMaxTokens = (int64_t)1 << 30;

ttt_status cuda_status(cudaError_t e) { return e == cudaSuccess ? TTT_OK : TTT_ERR_CUDA; }

}  // namespace

extern "C" {

const char* ttt_status_string(ttt_status s) {
  switch (s) {
    case TTT_OK: return "ok";
    case TTT_ERR_INVALID_ARG: return "invalid argument";
    case TTT_ERR_UNSUPPORTED_SHAPE: return "unsupported shape or option";
    case TTT_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case TTT_ERR_WORKSPACE: return "workspace missing or too small";
    case TTT_ERR_CUDA: return "CUDA runtime error";
    case TTT_ERR_DEVICE: return "a kernel gave up a bounded wait";
  }
  return "unknown status";
}

size_t ttt_update_workspace_bytes(const ttt_config* cfg, int64_t n_tokens) {
  if (check_cfg(cfg) != TTT_OK || n_tokens < 0 || n_tokens > kMaxTokens) return 0;
  return update_workspace(cfg, make_problem(cfg, n_tokens));
}

size_t ttt_shadow_bytes(const ttt_config* cfg) {
  if (check_cfg(cfg) != TTT_OK) return 0;
  return (size_t)(is_linear(cfg) ? 1 : 3) * cfg->heads * cfg->d * cfg->hidden * 2;
}

ttt_status ttt_update(const ttt_config* cfg, const float* W1, const float* W2, const float* W3,
                      const void* K, const void* V, const float* eta, int64_t n, float* W1_out,
                      float* W2_out, float* W3_out, void* shadow, void* workspace,
                      size_t workspace_bytes, ttt_stream_t stream) {
  ttt_status s = check_cfg(cfg);
  if (s != TTT_OK) return s;
  if (n < 0 || n > kMaxTokens) return TTT_ERR_INVALID_ARG;
  if (!W1 || !W1_out) return TTT_ERR_INVALID_ARG;
  if (!is_linear(cfg) && (!W2 || !W3 || !W2_out || !W3_out)) return TTT_ERR_INVALID_ARG;
  if (n > 0 && (!K || !V || !eta)) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {W1, W2, W3, K, V, eta, W1_out, W2_out, W3_out, shadow, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGNMENT;
  const Problem p = make_problem(cfg, n);
  const size_t need = update_workspace(cfg, p);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return TTT_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  auto* sh = static_cast<__nv_bfloat16_raw*>(shadow);
  if (is_linear(cfg))
    return cuda_status(ttt::linear_update(p, cfg->precision == TTT_PREC_BF16_TC, W1, K, V, eta,
                                          W1_out, sh, workspace, st));
  if (cfg->precision == TTT_PREC_FP32_CHECK)
    return cuda_status(ttt::f32_update(p, W1, W2, W3, static_cast<const float*>(K),
                                       static_cast<const float*>(V), eta, W1_out, W2_out, W3_out,
                                       sh, workspace, st));
  return cuda_status(
      ttt::tc_update(p, W1, W2, W3, K, V, eta, W1_out, W2_out, W3_out, sh, workspace, st));
}

ttt_status ttt_apply(const ttt_config* cfg, const float* W1, const float* W2, const float* W3,
                     const void* shadow, const void* Q, int64_t m, void* O,
                     ttt_stream_t stream) {
  ttt_status s = check_cfg(cfg);
  if (s != TTT_OK) return s;
  if (m < 0 || m > kMaxTokens) return TTT_ERR_INVALID_ARG;
  if (m > 0 && (!Q || !O)) return TTT_ERR_INVALID_ARG;
  if (cfg->precision == TTT_PREC_FP32_CHECK) {
    if (!W1 || (!is_linear(cfg) && (!W2 || !W3))) return TTT_ERR_INVALID_ARG;
  } else if (!shadow) {
    return TTT_ERR_INVALID_ARG;
  }
  const void* ptrs[] = {W1, W2, W3, shadow, Q, O};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGNMENT;
  const Problem p = make_problem(cfg, m);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (is_linear(cfg))
    return cuda_status(ttt::linear_apply(p, cfg->precision == TTT_PREC_BF16_TC, W1,
                                         static_cast<const __nv_bfloat16_raw*>(shadow), Q, O, st));
  if (cfg->precision == TTT_PREC_FP32_CHECK)
    return cuda_status(ttt::f32_apply(p, W1, W2, W3, static_cast<const float*>(Q),
                                      static_cast<float*>(O), st));
  return cuda_status(
      ttt::tc_apply(p, static_cast<const __nv_bfloat16_raw*>(shadow), Q, O, st));
}

ttt_status ttt_pack_shadow(const ttt_config* cfg, const float* W1, const float* W2,
                           const float* W3, void* shadow, ttt_stream_t stream) {
  ttt_status s = check_cfg(cfg);
  if (s != TTT_OK) return s;
  if (!W1 || !shadow || (!is_linear(cfg) && (!W2 || !W3))) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {W1, W2, W3, shadow};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGNMENT;
  if (is_linear(cfg)) W2 = W3 = nullptr;
  return cuda_status(ttt::pack_shadow(cfg->heads, cfg->d, cfg->hidden, W1, W2, W3,
                                      static_cast<__nv_bfloat16_raw*>(shadow),
                                      reinterpret_cast<cudaStream_t>(stream)));
}

ttt_status ttt_stream_step(const ttt_config* cfg, float* W1, float* W2, float* W3, void* shadow,
                           const void* K, const void* V, const float* eta, int64_t n,
                           const void* Q, int64_t m, void* O, void* workspace,
                           size_t workspace_bytes, ttt_stream_t stream) {
  ttt_status s = check_cfg(cfg);
  if (s != TTT_OK) return s;
  if (cfg->precision == TTT_PREC_BF16_TC && !shadow) return TTT_ERR_INVALID_ARG;
  if (m < 0 || m > kMaxTokens) return TTT_ERR_INVALID_ARG;
  if (m > 0 && (!Q || !O)) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {Q, O};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGNMENT;
  s = ttt_update(cfg, W1, W2, W3, K, V, eta, n, W1, W2, W3, shadow, workspace, workspace_bytes,
                 stream);
  if (s != TTT_OK) return s;
  return ttt_apply(cfg, W1, W2, W3, shadow, Q, m, O, stream);
}

ttt_status ttt_gate(const ttt_config* cfg, const void* Wg, const void* O_prime, int64_t m,
                    void* O, ttt_stream_t stream) {
  ttt_status s = check_cfg(cfg);
  if (s != TTT_OK) return s;
  if (m < 0 || m > kMaxTokens) return TTT_ERR_INVALID_ARG;
  if (!Wg) return TTT_ERR_INVALID_ARG;
  if (m > 0 && (!O_prime || !O)) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {Wg, O_prime, O};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGNMENT;
  const Problem p = make_problem(cfg, m);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cfg->precision == TTT_PREC_FP32_CHECK)
    return cuda_status(ttt::f32_gate(p, static_cast<const float*>(Wg),
                                     static_cast<const float*>(O_prime), static_cast<float*>(O),
                                     TTT_GATE_EPS, st));
  return cuda_status(ttt::tc_gate(p, Wg, O_prime, O, TTT_GATE_EPS, st));
}

int32_t ttt_update_splits(const ttt_config* cfg, int64_t n_tokens) {
  if (check_cfg(cfg) != TTT_OK || n_tokens < 0 || n_tokens > kMaxTokens) return 0;
  const Problem p = make_problem(cfg, n_tokens);
  if (is_linear(cfg)) return ttt::linear_split_plan(p).S;
  return cfg->precision == TTT_PREC_FP32_CHECK ? ttt::f32_split_plan(p).S
                                               : ttt::tc_split_plan(p).S;
}

size_t ttt_partial_floats(const ttt_config* cfg) {
  if (check_cfg(cfg) != TTT_OK) return 0;
  return (size_t)(is_linear(cfg) ? 1 : 3) * cfg->heads * cfg->d * cfg->hidden;
}

size_t ttt_finish_workspace_bytes(const ttt_config* cfg) {
  if (check_cfg(cfg) != TTT_OK) return 0;
  const Problem p = make_problem(cfg, 1);
  const size_t scratch = ttt::align_up((size_t)p.H * (2 * p.hid + p.d) * 2 * sizeof(double), 1024);
  return scratch + ttt::ns_workspace_bytes(p);
}

ttt_status ttt_update_partial(const ttt_config* cfg, const float* W1, const float* W2,
                              const float* W3, const void* K, const void* V, const float* eta,
                              int64_t n, float* partial, void* workspace, size_t workspace_bytes,
                              ttt_stream_t stream) {
  ttt_status s = check_cfg(cfg);
  if (s != TTT_OK) return s;
  if (n < 0 || n > kMaxTokens) return TTT_ERR_INVALID_ARG;
  if (!W1 || !partial || (!is_linear(cfg) && (!W2 || !W3))) return TTT_ERR_INVALID_ARG;
  if (n > 0 && (!K || !V || !eta)) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {W1, W2, W3, K, V, eta, partial, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGNMENT;
  const Problem p = make_problem(cfg, n);
  const bool tc = cfg->precision == TTT_PREC_BF16_TC;
  const size_t need = update_workspace(cfg, p);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return TTT_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (is_linear(cfg))
    return cuda_status(ttt::linear_update(p, tc, W1, K, V, eta, nullptr, nullptr, workspace, st,
                                          partial));
  if (!tc)
    return cuda_status(ttt::f32_update(p, W1, W2, W3, static_cast<const float*>(K),
                                       static_cast<const float*>(V), eta, nullptr, nullptr,
                                       nullptr, nullptr, workspace, st, partial));
  return cuda_status(ttt::tc_update(p, W1, W2, W3, K, V, eta, nullptr, nullptr, nullptr, nullptr,
                                    workspace, st, partial));
}

ttt_status ttt_update_finish(const ttt_config* cfg, const float* W1, const float* W2,
                             const float* W3, const float* partials, int32_t ranks,
                             float* W1_out, float* W2_out, float* W3_out, void* shadow,
                             void* workspace, size_t workspace_bytes, ttt_stream_t stream) {
  ttt_status s = check_cfg(cfg);
  if (s != TTT_OK) return s;
  if (ranks < 1 || ranks > 65536) return TTT_ERR_INVALID_ARG;
  if (!W1 || !partials || !W1_out) return TTT_ERR_INVALID_ARG;
  if (!is_linear(cfg) && (!W2 || !W3 || !W2_out || !W3_out)) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {W1, W2, W3, partials, W1_out, W2_out, W3_out, shadow, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGNMENT;
  const size_t need = ttt_finish_workspace_bytes(cfg);
  if (workspace == nullptr || workspace_bytes < need) return TTT_ERR_WORKSPACE;
  // n only gates the Newton-Schulz stage (skipped for an empty update); the
  // partials carry the tokens.
  const Problem p = make_problem(cfg, 1);
  char* ws = static_cast<char*>(workspace);
  float* scratch = reinterpret_cast<float*>(ws);
  void* ns_ws = ws + ttt::align_up((size_t)p.H * (2 * p.hid + p.d) * 2 * sizeof(double), 1024);
  return cuda_status(ttt::ns_then_renorm(p, ranks, partials, ns_ws,
                                         cfg->precision == TTT_PREC_BF16_TC, W1, W2, W3, W1_out,
                                         W2_out, W3_out, static_cast<__nv_bfloat16_raw*>(shadow),
                                         scratch, reinterpret_cast<cudaStream_t>(stream)));
}

ttt_status ttt_chunked(const ttt_config* cfg, float* W1, float* W2, float* W3, void* shadow,
                       const void* K, const void* V, const float* eta, const void* Q,
                       int64_t n, int64_t chunk, int32_t order, const uint8_t* update_mask,
                       void* O, void* workspace, size_t workspace_bytes, ttt_stream_t stream) {
  ttt_status s = check_cfg(cfg);
  if (s != TTT_OK) return s;
  if (n < 0 || n > kMaxTokens || chunk < 1) return TTT_ERR_INVALID_ARG;
  if (order != TTT_ORDER_UPDATE_THEN_APPLY && order != TTT_ORDER_APPLY_THEN_UPDATE)
    return TTT_ERR_INVALID_ARG;
  if (!W1 || (!is_linear(cfg) && (!W2 || !W3))) return TTT_ERR_INVALID_ARG;
  const bool tc = cfg->precision == TTT_PREC_BF16_TC;
  if (tc && !shadow) return TTT_ERR_INVALID_ARG;
  if (n == 0) return TTT_OK;
  if (!K || !V || !eta || !Q || !O) return TTT_ERR_INVALID_ARG;
  const void* ptrs[] = {W1, W2, W3, shadow, K, V, eta, Q, O, workspace};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return TTT_ERR_ALIGNMENT;
  if ((chunk * cfg->heads) % 4 != 0) return TTT_ERR_ALIGNMENT;
  const int64_t first = chunk < n ? chunk : n;
  const int64_t nchunks = (n + chunk - 1) / chunk;
  bool any_update = false;
  for (int64_t i = 0; i < nchunks; ++i) any_update |= update_mask == nullptr || update_mask[i] != 0;
  if (any_update) {
    const Problem p = make_problem(cfg, first);
    const size_t need = update_workspace(cfg, p);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return TTT_ERR_WORKSPACE;
  }
  // Every chunk's pointers keep the base alignment (token rows are multiples
  // of 128 bytes, eta rows start at multiples of 16 bytes), and no chunk is
  // longer than the first, so the per-chunk calls below pass their checks.
  const size_t tok = (size_t)cfg->heads * cfg->d * (tc ? 2 : 4);
  const char* k8 = static_cast<const char*>(K);
  const char* v8 = static_cast<const char*>(V);
  const char* q8 = static_cast<const char*>(Q);
  char* o8 = static_cast<char*>(O);
  const bool first_is_apply = order == TTT_ORDER_APPLY_THEN_UPDATE ||
                              (update_mask != nullptr && update_mask[0] == 0);
  if (tc && first_is_apply) {
    s = ttt_pack_shadow(cfg, W1, W2, W3, shadow, stream);
    if (s != TTT_OK) return s;
  }
  for (int64_t i = 0; i < nchunks; ++i) {
    const int64_t s0 = i * chunk, len = (s0 + chunk <= n ? chunk : n - s0);
    const bool upd = update_mask == nullptr || update_mask[i] != 0;
    if (order == TTT_ORDER_APPLY_THEN_UPDATE) {
      s = ttt_apply(cfg, W1, W2, W3, shadow, q8 + s0 * tok, len, o8 + s0 * tok, stream);
      if (s != TTT_OK) return s;
    }
    if (upd) {
      s = ttt_update(cfg, W1, W2, W3, k8 + s0 * tok, v8 + s0 * tok, eta + s0 * cfg->heads, len,
                     W1, W2, W3, shadow, workspace, workspace_bytes, stream);
      if (s != TTT_OK) return s;
    }
    if (order == TTT_ORDER_UPDATE_THEN_APPLY) {
      s = ttt_apply(cfg, W1, W2, W3, shadow, q8 + s0 * tok, len, o8 + s0 * tok, stream);
      if (s != TTT_OK) return s;
    }
  }
  return TTT_OK;
}

ttt_status ttt_selftest_wait_timeout(int64_t limit_cycles, ttt_stream_t stream) {
  if (limit_cycles < 1 || limit_cycles > ((int64_t)1 << 31)) return TTT_ERR_INVALID_ARG;
  return cuda_status(
      ttt::selftest_wait_timeout((long long)limit_cycles, reinterpret_cast<cudaStream_t>(stream)));
}

ttt_status ttt_check_device_error(ttt_stream_t stream, int32_t* code) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return TTT_ERR_CUDA;
  int v = 0;
  if (ttt::read_and_clear_device_error(&v) != cudaSuccess) return TTT_ERR_CUDA;
  if (code) *code = v;
  return v != 0 ? TTT_ERR_DEVICE : TTT_OK;
}

}  // extern "C"
