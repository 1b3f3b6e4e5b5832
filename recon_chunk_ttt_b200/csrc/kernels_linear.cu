// Linear fast weights (67656.sbs reading notes "ZipMap：基于 Test-Time Training 的线性时间
// 有状态 3D 重建", section "为什么它像 attention（线性情形的直观推导）"): with
// f_W(k) = W k, W ∈ R^{d×d} per head, the virtual loss L = -Σ_i η_i (W k_i)^T v_i
// has the gradient g = -Σ_i η_i v_i k_i^T, so one step gives
//   Ŵ = renorm(W + Σ_i η_i v_i k_i^T)        (renorm off: the closed form)
// and the read is o = Ŵ q = W q + Σ_i η_i v_i (k_i^T q), an un-normalised
// linear attention over the chunk.
//
// This mode exists to check the layer's machinery against that closed form;
// it is not the benchmarked path.  Its two contractions run on CUDA cores
// with fp32 arithmetic in both precisions (BF16_TC reads bf16 tokens and the
// bf16 weight shadow and writes bf16 outputs; FP32_CHECK reads and writes
// fp32), with a fixed token order inside each split, so results are bitwise
// reproducible.

#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace ttt {
namespace {

constexpr int kT = 16;  // tokens (update) or contraction elements (apply) per step
constexpr int kB = 64;  // output tile edge

__device__ __forceinline__ float ld_tok(const float* p) { return *p; }
__device__ __forceinline__ float ld_tok(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_tok(float* p, float v) { *p = v; }
__device__ __forceinline__ void st_tok(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// Split s of head h: P_s[i][j] = Σ_{t in split s} η_t v_t[i] k_t[j] over its
// tokens in increasing order.  grid = ((d/64)^2, H, S), 256 threads, a 4x4
// block of outputs per thread.
template <typename T>
__global__ void __launch_bounds__(256) linear_grad_kernel(const T* __restrict__ K,
                                                          const T* __restrict__ V,
                                                          const float* __restrict__ eta,
                                                          int64_t n, int H, int d, int64_t chunk,
                                                          float* __restrict__ partials) {
  __shared__ float sV[kT][kB + 4], sK[kT][kB + 4];
  const int tiles = d / kB;
  const int i0 = (blockIdx.x / tiles) * kB, j0 = (blockIdx.x % tiles) * kB;
  const int h = blockIdx.y, s = blockIdx.z;
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const int64_t ld = (int64_t)H * d;
  const int64_t t0 = (int64_t)s * chunk;
  const int64_t t1 = t0 + chunk < n ? t0 + chunk : n;
  float acc[4][4] = {};
  for (int64_t tb = t0; tb < t1; tb += kT) {
    for (int e = tid; e < kT * kB; e += 256) {
      const int t = e / kB, c = e % kB;
      const int64_t tok = tb + t;
      float vv = 0.f, kv = 0.f;
      if (tok < t1) {
        vv = eta[tok * H + h] * ld_tok(V + tok * ld + (int64_t)h * d + i0 + c);
        kv = ld_tok(K + tok * ld + (int64_t)h * d + j0 + c);
      }
      sV[t][c] = vv;
      sK[t][c] = kv;
    }
    __syncthreads();
#pragma unroll
    for (int t = 0; t < kT; ++t) {
      float a[4], b[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a[q] = sV[t][ty * 4 + q];
        b[q] = sK[t][tx * 4 + q];
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(a[x], b[y], acc[x][y]);
    }
    __syncthreads();
  }
  float* P = partials + ((size_t)s * H + h) * (size_t)d * d;
#pragma unroll
  for (int x = 0; x < 4; ++x)
    *reinterpret_cast<float4*>(P + (size_t)(i0 + ty * 4 + x) * d + j0 + tx * 4) =
        make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
}

// O[t][h*d + i] = Σ_j W[h][i][j] q[t][h*d + j].  grid = (ceil(m/64), d/64, H),
// 256 threads, a 4 (tokens) x 4 (outputs) block per thread.
template <typename T, typename WT>
__global__ void __launch_bounds__(256) linear_apply_kernel(const WT* __restrict__ W,
                                                           const T* __restrict__ Q, int64_t m,
                                                           int H, int d, T* __restrict__ O) {
  __shared__ float sQ[kT][kB + 4], sW[kT][kB + 4];
  const int64_t t0 = (int64_t)blockIdx.x * kB;
  const int i0 = blockIdx.y * kB, h = blockIdx.z;
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const int64_t ld = (int64_t)H * d;
  const WT* Wh = W + (size_t)h * d * d;
  float acc[4][4] = {};
  for (int j0 = 0; j0 < d; j0 += kT) {
    for (int e = tid; e < kT * kB; e += 256) {
      const int r = e / kT, c = e % kT;  // r: token (Q) or output row (W); c: contraction index
      const int64_t tok = t0 + r;
      sQ[c][r] = tok < m ? ld_tok(Q + tok * ld + (int64_t)h * d + j0 + c) : 0.f;
      sW[c][r] = ld_tok(Wh + (size_t)(i0 + r) * d + j0 + c);
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < kT; ++c) {
      float a[4], b[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a[q] = sQ[c][ty * 4 + q];
        b[q] = sW[c][tx * 4 + q];
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(a[x], b[y], acc[x][y]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    const int64_t tok = t0 + ty * 4 + x;
    if (tok >= m) continue;
#pragma unroll
    for (int y = 0; y < 4; ++y) st_tok(O + tok * ld + (int64_t)h * d + i0 + tx * 4 + y, acc[x][y]);
  }
}

}  // namespace

SplitPlan linear_split_plan(const Problem& p) {
  // about one wave of (d/64)^2 x H tile blocks per split, at least 512 tokens
  // per split
  const int per = (p.d / kB) * (p.d / kB) * p.H;
  int S = 148 * 2 / per;
  if (S < 1) S = 1;
  const int64_t max_s = (p.n + 511) / 512;
  if (S > max_s) S = (int)(max_s < 1 ? 1 : max_s);
  int64_t chunk = (p.n + S - 1) / S;
  chunk = (chunk + kT - 1) / kT * kT;
  if (chunk < kT) chunk = kT;
  if (p.n > 0) S = (int)((p.n + chunk - 1) / chunk);
  return {S, chunk};
}

size_t linear_workspace_bytes(const Problem& p) {
  const SplitPlan sp = linear_split_plan(p);
  return align_up((size_t)sp.S * p.H * p.d * p.d * 4, 1024) +
         align_up((size_t)p.H * p.d * 2 * 8, 1024);
}

cudaError_t linear_update(const Problem& p, bool bf16_tokens, const float* W, const void* K,
                          const void* V, const float* eta, float* Wo,
                          __nv_bfloat16_raw* shadow, void* ws, cudaStream_t st,
                          float* partial_out) {
  const SplitPlan sp = linear_split_plan(p);
  float* partials = static_cast<float*>(ws);
  float* scratch = reinterpret_cast<float*>(static_cast<char*>(ws) +
                                            align_up((size_t)sp.S * p.H * p.d * p.d * 4, 1024));
  const size_t count = (size_t)p.H * p.d * p.d;
  if (p.n > 0) {
    const dim3 grid((unsigned)((p.d / kB) * (p.d / kB)), (unsigned)p.H, (unsigned)sp.S);
    TraceScope ts("linear_grad", st);
    if (bf16_tokens)
      linear_grad_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
          static_cast<const __nv_bfloat16*>(K), static_cast<const __nv_bfloat16*>(V), eta, p.n,
          p.H, p.d, sp.chunk, partials);
    else
      linear_grad_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(K),
                                                      static_cast<const float*>(V), eta, p.n,
                                                      p.H, p.d, sp.chunk, partials);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  } else {
    const cudaError_t e = cudaMemsetAsync(partials, 0, (size_t)sp.S * count * 4, st);
    if (e != cudaSuccess) return e;
  }
  if (partial_out != nullptr) return sum_splits(sp.S, count, partials, partial_out, st);
  return reduce_renorm(p, sp.S, partials, W, nullptr, nullptr, Wo, nullptr, nullptr, shadow,
                       scratch, st);
}

cudaError_t linear_apply(const Problem& p, bool bf16, const float* W,
                         const __nv_bfloat16_raw* shadow, const void* Q, void* O,
                         cudaStream_t st) {
  if (p.n == 0) return cudaSuccess;
  const dim3 grid((unsigned)((p.n + kB - 1) / kB), (unsigned)(p.d / kB), (unsigned)p.H);
  TraceScope ts("linear_apply", st);
  if (bf16)
    linear_apply_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(shadow), static_cast<const __nv_bfloat16*>(Q),
        p.n, p.H, p.d, static_cast<__nv_bfloat16*>(O));
  else
    linear_apply_kernel<float, float><<<grid, 256, 0, st>>>(
        W, static_cast<const float*>(Q), p.n, p.H, p.d, static_cast<float*>(O));
  return cudaGetLastError();
}

}  // namespace ttt
