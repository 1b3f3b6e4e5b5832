/*
 * recon_chunk_ttt_b200 — C ABI of the ZipMap global large-chunk TTT layer on
 * B200 (sm_100a).
 *
 * The layer (kimjy99, "[논문리뷰] ZipMap: Linear-Time Stateful 3D
 * Reconstruction via Test-Time Training", section 2 "Feature Backbone"):
 *
 *   f_W(x) = W2 [ SiLU(W1 x) ⊙ (W3 x) ]                          (Eq. 1)
 *   L_i    = -f_W(k_i)^T v_i                                      (Eq. 2)
 *   g      = ∇_W Σ_i η_i L_i     (over every token of the chunk)   (Eq. 3)
 *   Ŵ      = ‖W‖ · (W - g) / ‖W - g‖   (L2 renormalisation, the update
 *                                       equations after Eq. 3)
 *   o_i    = f_Ŵ(q_i)            (apply, to image or ray-map queries)
 *
 * and, for streaming (section 3 "Streaming Reconstruction"), the same update
 * with the tokens of one frame at a time, the state carried across calls.
 * The renormalisation axis is row-wise (each row of W1, W3 of length d, each
 * row of W2 of length hidden, rescaled to its pre-update norm); "frobenius"
 * (one norm per matrix per head) and "off" are switches.
 *
 * Newton–Schulz (same section, the update after Eq. 3: Δ ← NewtonSchulz(g),
 * following the Muon optimizer; then Ŵ = ‖W‖ · (W − Δ)/‖W − Δ‖) is a switch,
 * ns_steps (0 = off, the layer above).  The page gives neither the polynomial
 * nor the step count; with ns_steps = k > 0 each of g1, g2, g3 of each head is
 * replaced by k steps of Muon's quintic iteration on X0 = g/‖g‖_F:
 *   X ← a X + (b A + c A²) X,  A = X Xᵀ,  (a, b, c) = (3.4445, −4.7750, 2.0315),
 * worked on the wide (d × hidden) orientation; g = 0 gives Δ = 0.  In
 * BF16_TC mode its GEMMs run on the tensor cores with each fp32 operand split
 * into two bf16 parts (hi + lo, three products), the iterate kept in fp32.
 *
 * Conventions shared by every entry point
 *  - All pointers except `cfg` are DEVICE pointers on the current CUDA device,
 *    owned by the caller; the library allocates no device memory and keeps no
 *    state between calls apart from one device error word per device and the
 *    optional tracing totals (ttt_trace_enable).
 *  - Every call is asynchronous on `stream` (NULL = the legacy default
 *    stream); arguments are validated on the host before anything is
 *    enqueued, so an error status means nothing was launched.
 *  - The update, reduce/renorm and apply kernels are launched as
 *    programmatic dependents (CUDA programmatic dependent launch): each
 *    waits for the complete, visible results of the work ahead of it on the
 *    stream before reading anything, and lets the next kernel on the stream
 *    start its launch early.  A caller's kernel that follows on the same
 *    stream and is itself launched with programmatic stream serialization
 *    must wait for its dependency (cudaGridDependencySynchronize) before
 *    reading this library's outputs; any other following work is ordered
 *    as usual.
 *  - Layouts are dense, row-major, per head h = 0..H-1:
 *        W1, W3 : float [H][hidden][d]      W2 : float [H][d][hidden]
 *        K, V, Q: [n][H*d] token-major, bf16 (precision BF16_TC) or
 *                 float (precision FP32_CHECK); head h is columns h*d..h*d+d-1
 *        eta    : float [n][H]
 *        O      : [m][H*d], bf16 (BF16_TC) or float (FP32_CHECK)
 *        shadow : bf16 copies of Ŵ for the tensor-core apply, in the same
 *                 layout as W1, W3, W2 (W1 block, then W3, then W2);
 *                 ttt_shadow_bytes() bytes.
 *  - Device pointers must be 16-byte aligned (tensor-memory-access rule).
 *  - Supported shapes: (d, hidden) = (64, 128) or (256, 512), heads >= 1
 *    (linear mode: (64, 64) or (256, 256)).
 *  - n = 0 or eta = 0 gives Ŵ = W.  Outputs may alias the weight inputs
 *    (in-place update); K, V, Q, eta and O must not alias outputs.
 *  - Results are deterministic run to run (fixed-order reductions, no
 *    atomics in any sum).
 */
#ifndef RECON_CHUNK_TTT_H
#define RECON_CHUNK_TTT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* ttt_stream_t;

typedef enum {
  TTT_OK = 0,
  TTT_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum   */
  TTT_ERR_UNSUPPORTED_SHAPE = 2, /* (d, hidden) not supported               */
  TTT_ERR_ALIGNMENT = 3,         /* a pointer is not 16-byte aligned        */
  TTT_ERR_WORKSPACE = 4,         /* workspace missing or too small          */
  TTT_ERR_CUDA = 5,              /* a CUDA runtime call failed              */
  TTT_ERR_DEVICE = 6             /* a kernel gave up a bounded wait         */
} ttt_status;

/* Fast-weight form.  TTT_MLP_SWIGLU: the layer above.  TTT_MLP_LINEAR:
 * f_W(k) = W k with one d x d matrix per head (67656.sbs reading notes,
 * section "为什么它像 attention（线性情形的直观推导）"), for which one step has
 * the closed form Ŵ = W + Σ_i η_i v_i k_i^T (before the renormalisation) and
 * the read o = Ŵ q is an un-normalised linear attention.  In linear mode
 * hidden must equal d, ns_steps must be 0, W is passed as W1 ([H][d][d],
 * row = output), W2 and W3 (and W2_out, W3_out) are unused and may be NULL,
 * the shadow holds the one bf16 matrix (H * d * d * 2 bytes) and partials
 * are [H][1][d*d] holding Σ η v k^T (= -g).  Its two contractions run on
 * CUDA cores with fp32 arithmetic in both precisions (BF16_TC reads bf16
 * tokens and the bf16 shadow and writes bf16 outputs); it is a reference
 * mode for that closed form, not the benchmarked layer. */
enum { TTT_MLP_SWIGLU = 0, TTT_MLP_LINEAR = 1 };
enum { TTT_RENORM_OFF = 0, TTT_RENORM_ROW = 1, TTT_RENORM_FROB = 2 };
enum { TTT_PREC_BF16_TC = 0, TTT_PREC_FP32_CHECK = 1 };
enum { TTT_MAX_NS_STEPS = 32 };

typedef struct {
  int32_t heads;     /* H, number of independent fast-weight MLPs          */
  int32_t d;         /* head dimension (64 or 256)                         */
  int32_t hidden;    /* fast-weight hidden width (128 or 512)              */
  int32_t mlp;       /* TTT_MLP_SWIGLU or TTT_MLP_LINEAR                   */
  int32_t renorm;    /* TTT_RENORM_*                                       */
  int32_t ns_steps;  /* Newton–Schulz steps on g: 0 (off) .. TTT_MAX_NS_STEPS */
  int32_t precision; /* TTT_PREC_BF16_TC: bf16 tensor-core operands, fp32
                        accumulation; TTT_PREC_FP32_CHECK: fp32 CUDA-core
                        arithmetic throughout                              */
} ttt_config;

/* Human-readable name of a status code (static string). */
const char* ttt_status_string(ttt_status s);

/* Bytes of device workspace ttt_update / ttt_stream_step need for n tokens
 * (0 if the config is invalid). */
size_t ttt_update_workspace_bytes(const ttt_config* cfg, int64_t n_tokens);

/* Bytes of the bf16 weight shadow (3 * H * d * hidden * 2; linear mode
 * H * d * d * 2). */
size_t ttt_shadow_bytes(const ttt_config* cfg);

/* Number of token splits S the update of n tokens reduces: the gradient is
 * accumulated as S fp32 partials over contiguous token ranges (a function of
 * cfg and n only), summed in increasing split order before the
 * renormalisation.  The workspace holds them.  0 if the config is invalid. */
int32_t ttt_update_splits(const ttt_config* cfg, int64_t n_tokens);

/*
 * One TTT update of all heads (Eq. 1–3 and the renormalisation above):
 *   g = ∇_W Σ_{i<n} η_i (−f_W(k_i)^T v_i),  Ŵ = renorm(W − Δ),
 *   Δ = g (ns_steps = 0) or NewtonSchulz(g) (ns_steps > 0).
 * Inputs W1, W2, W3 (fp32), K, V, eta for n >= 0 tokens.  Writes Ŵ to
 * W1_out, W2_out, W3_out (fp32, may equal the inputs) and, when `shadow` is
 * not NULL, bf16 copies of Ŵ to `shadow` for ttt_apply.
 * `workspace` must hold ttt_update_workspace_bytes(cfg, n) bytes (it may be
 * NULL when that is 0); its contents need no initialisation.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, ALIGNMENT, WORKSPACE, CUDA.
 */
ttt_status ttt_update(const ttt_config* cfg,
                      const float* W1, const float* W2, const float* W3,
                      const void* K, const void* V, const float* eta, int64_t n,
                      float* W1_out, float* W2_out, float* W3_out, void* shadow,
                      void* workspace, size_t workspace_bytes, ttt_stream_t stream);

/*
 * Apply (read) the fast weights to m >= 0 queries: O[i] = f_Ŵ(Q[i]) per head
 * (section 2 of the review: o'_i = f_Ŵ(q_i); ray-map target queries use the
 * same call).  BF16_TC reads `shadow` (bf16 Ŵ, from ttt_update or
 * ttt_pack_shadow) and ignores W1..W3 (may be NULL); FP32_CHECK reads W1..W3
 * and ignores `shadow`.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, ALIGNMENT, CUDA.
 */
ttt_status ttt_apply(const ttt_config* cfg,
                     const float* W1, const float* W2, const float* W3,
                     const void* shadow, const void* Q, int64_t m, void* O,
                     ttt_stream_t stream);

/* Write bf16 copies of W1, W2, W3 into `shadow` (for ttt_apply on weights
 * that did not come out of ttt_update). */
ttt_status ttt_pack_shadow(const ttt_config* cfg,
                           const float* W1, const float* W2, const float* W3,
                           void* shadow, ttt_stream_t stream);

/*
 * One streaming step (section 3 of the review, the per-frame TTTUpdate):
 * updates the state W1, W2, W3 IN PLACE with the n tokens of one frame, then
 * applies the new state to that frame's m queries, writing O.  `shadow` is
 * required for BF16_TC (it receives the bf16 copy of the new state) and may
 * be NULL for FP32_CHECK.  Workspace as for ttt_update(cfg, n).
 */
ttt_status ttt_stream_step(const ttt_config* cfg,
                           float* W1, float* W2, float* W3, void* shadow,
                           const void* K, const void* V, const float* eta, int64_t n,
                           const void* Q, int64_t m, void* O,
                           void* workspace, size_t workspace_bytes, ttt_stream_t stream);

/*
 * Synchronise `stream`, then read and clear this device's error word.  A
 * kernel that gives up a bounded wait (it never spins without a limit) sets
 * the word and returns early; such a call's outputs are undefined.
 * Returns TTT_OK, TTT_ERR_DEVICE (and *code = the kernel's reason, if code
 * is not NULL) or TTT_ERR_CUDA.
 */
ttt_status ttt_check_device_error(ttt_stream_t stream, int32_t* code);

/*
 * Failure-detection self-test (no counterpart on the pages): launches one
 * block whose thread waits, through the same bounded mbarrier wait the
 * kernels use, on a barrier nothing completes.  After limit_cycles SM cycles
 * (1 .. 2^31) the wait gives up, writes TTT_DEVICE_ERR_SELFTEST into the
 * device error word and the kernel returns; the next ttt_check_device_error
 * then returns TTT_ERR_DEVICE with that code, and the context stays usable.
 * Nothing traps or hangs.
 */
enum { TTT_DEVICE_ERR_SELFTEST = 7 };
ttt_status ttt_selftest_wait_timeout(int64_t limit_cycles, ttt_stream_t stream);

/*
 * Gated output unit (kimjy99 review, section 2 "Feature Backbone", the last
 * equation): o = RMSNorm(o') ⊙ SiLU(W_g o'), applied per head to the layer
 * output o' (e.g. ttt_apply's O).  The page does not say whether the unit
 * spans heads; heads being independent here, it is read per head:
 *   RMSNorm(x) = x / sqrt(mean_j x_j² + TTT_GATE_EPS)   (no learned gain)
 *   W_g: [H][d][d], row = output; bf16 (BF16_TC) or float (FP32_CHECK)
 *   O_prime, O: [m][H*d], the token type of the precision; O may equal
 *   O_prime (in place).
 * BF16_TC: W_g o' on the tensor cores (fp32 accumulation), RMS and gate in
 * fp32, o rounded to bf16.
 */
#define TTT_GATE_EPS 1e-6f
ttt_status ttt_gate(const ttt_config* cfg, const void* Wg, const void* O_prime, int64_t m,
                    void* O, ttt_stream_t stream);

/*
 * Token-sharded update across ranks (one chunk's tokens split over several
 * GPUs; the pages describe one GPU, this is the data-parallel form of the
 * same sum).  Eq. 3's g is a sum over tokens, so each rank reduces its own
 * tokens to a partial and the ranks exchange partials (an all-gather, e.g.
 * NCCL over NVLink, done by the caller); every rank then forms the same Ŵ.
 *
 * ttt_update_partial: the gradient partial of this rank's n tokens (weights
 *   W, tokens K, V, eta as in ttt_update) into `partial`, fp32, layout
 *   [H][3][hidden*d]: block 0 = g1 ([hidden][d]), block 1 = g3 ([hidden][d]),
 *   block 2 = −g2 ([d][hidden]); ttt_partial_floats(cfg) floats.  Partials add
 *   elementwise.  Workspace: ttt_update_workspace_bytes(cfg, n).  n = 0 gives
 *   zeros.
 * ttt_update_finish: Ŵ from `ranks` partials stored one after another
 *   ([ranks][H][3][hidden*d]), summed in rank order in fp64 (so the result
 *   does not depend on which rank computes it, and all ranks agree bitwise),
 *   then NewtonSchulz (cfg.ns_steps > 0) and the renormalisation as in
 *   ttt_update, against the pre-update W.  Outputs and shadow as in
 *   ttt_update (may alias W).  Workspace: ttt_finish_workspace_bytes(cfg).
 */
size_t ttt_partial_floats(const ttt_config* cfg);
size_t ttt_finish_workspace_bytes(const ttt_config* cfg);
ttt_status ttt_update_partial(const ttt_config* cfg, const float* W1, const float* W2,
                              const float* W3, const void* K, const void* V, const float* eta,
                              int64_t n, float* partial, void* workspace, size_t workspace_bytes,
                              ttt_stream_t stream);
ttt_status ttt_update_finish(const ttt_config* cfg, const float* W1, const float* W2,
                             const float* W3, const float* partials, int32_t ranks,
                             float* W1_out, float* W2_out, float* W3_out, void* shadow,
                             void* workspace, size_t workspace_bytes, ttt_stream_t stream);

/*
 * LaCT chunked orderings (mhpn.cn survey of TTSA3R / LaCT / ZipMap / LoGeR,
 * part "二、LaCT", "3应用场景"): the n tokens are cut into consecutive chunks of
 * `chunk` tokens (the last one shorter), and chunk i = tokens
 * [i*chunk, min(n, (i+1)*chunk)) is processed in order:
 *   TTT_ORDER_UPDATE_THEN_APPLY (block-causal): W <- U(W; chunk i) if the
 *       chunk updates, then O[chunk i] = f_W(Q[chunk i]);
 *   TTT_ORDER_APPLY_THEN_UPDATE (shifted block-causal): O[chunk i] =
 *       f_W(Q[chunk i]) with the state before the chunk, then W <- U(W; chunk i)
 *       if the chunk updates.
 * U is the update of ttt_update (with cfg's renorm and ns_steps), in place.
 * `update_mask` is a HOST array of ceil(n/chunk) bytes (nonzero = the chunk
 * updates) or NULL (every chunk updates); updating only chosen chunks gives the
 * cross-chunk causal pattern.  One chunk with APPLY_THEN_UPDATE is LaCT's
 * fully bidirectional pattern; one chunk with UPDATE_THEN_APPLY is the ZipMap
 * layer, and frame-sized chunks its streaming recurrence.
 *  - Arguments as in ttt_stream_step, with Q and O for the same n tokens
 *    (each token has a query): K, V, Q [n][H*d], eta [n][H], O [n][H*d].
 *  - BF16_TC: `shadow` is required; when the first operation is an apply it
 *    is first packed from W (the caller's contents do not matter).
 *    FP32_CHECK: `shadow` may be NULL.
 *  - chunk >= 1 and chunk * heads a multiple of 4 (every chunk's eta rows
 *    then start 16-byte aligned); workspace: ttt_update_workspace_bytes(cfg,
 *    min(chunk, n)).  Every argument is checked before anything is enqueued.
 */
enum { TTT_ORDER_UPDATE_THEN_APPLY = 0, TTT_ORDER_APPLY_THEN_UPDATE = 1 };
ttt_status ttt_chunked(const ttt_config* cfg, float* W1, float* W2, float* W3, void* shadow,
                       const void* K, const void* V, const float* eta, const void* Q,
                       int64_t n, int64_t chunk, int32_t order, const uint8_t* update_mask,
                       void* O, void* workspace, size_t workspace_bytes, ttt_stream_t stream);

/*
 * Allocation-free streaming step (the pages have no counterpart: this is a
 * deployment aid).  Same arguments and result as ttt_stream_step() minus the
 * workspace: the scratch is a fixed TTT_STATIC_SCRATCH_BYTES device array
 * inside the library, for callers that cannot allocate device memory when a
 * frame arrives (fixed memory budgets, allocator owned by another runtime, no
 * cudaMalloc after start-up).  The call allocates nothing.
 *  - Returns TTT_ERR_WORKSPACE, before launching anything, when
 *    ttt_update_workspace_bytes(cfg, n) exceeds TTT_STATIC_SCRATCH_BYTES.
 *    The limit depends on the configuration.  BF16_TC keeps the update's
 *    intermediates on chip, so its workspace stops growing with n: with 4
 *    heads of d = 256, hidden 512 every n fits (25.2 MB with ns_steps = 0,
 *    69.3 MB with ns_steps > 0); for every n, up to 31 such heads fit with
 *    ns_steps = 0 and 6 with ns_steps > 0.  FP32_CHECK keeps per-token
 *    intermediates: 4 heads of d = 256 fit up to 3,836 tokens per call with
 *    ns_steps = 0 and 2,044 with ns_steps > 0 (one 518 x 518 frame is 1,374
 *    tokens).
 *  - Every GPU that loads the library may hold the array until exit.
 *  - All calls on a device share the array and it keeps the last call's
 *    contents (nothing in it has to start at zero); calls that can overlap on
 *    the GPU race on it and must be serialised by the caller.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) and caches it with the id of the device's current
 *    context; a call after the context changed (cudaDeviceReset, or the
 *    primary context released and created again) looks it up anew.  Make
 *    such a call (the first on each device, and the first after a reset)
 *    before any stream capture.
 */
#define TTT_STATIC_SCRATCH_BYTES ((size_t)96 << 20)
ttt_status ttt_stream_step_static(const ttt_config* cfg,
                                  float* W1, float* W2, float* W3, void* shadow,
                                  const void* K, const void* V, const float* eta, int64_t n,
                                  const void* Q, int64_t m, void* O, ttt_stream_t stream);

/*
 * Tracing.  With tracing on, every kernel launch of the library is bracketed
 * by two CUDA events on the caller's stream (host-side state: an event pool
 * and per-kernel totals, guarded by a mutex).  ttt_trace_read synchronises
 * the recorded events, adds their elapsed times to per-kernel totals and
 * copies up to `capacity` entries (name, launches, total milliseconds) into
 * `entries`; *count receives the number of kernel names seen.  reset != 0
 * clears the totals after reading.  Off by default.
 */
typedef struct {
  char name[32];
  int64_t launches;
  double total_ms;
} ttt_trace_entry;

ttt_status ttt_trace_enable(int32_t on);
ttt_status ttt_trace_read(ttt_trace_entry* entries, int32_t capacity, int32_t* count,
                          int32_t reset);

#ifdef __cplusplus
}
#endif

#endif /* RECON_CHUNK_TTT_H */
