// fp32 CUDA-core "check mode" of the TTT update and apply: no tensor cores,
// no TF32, fp32 arithmetic with fixed-order reductions.  Used to check the
// layer against the fp64 oracle at 1e-5 and as the baseline the tensor-core
// path is compared with.
//
// Math per head (kimjy99 ZipMap review, section 2, Eq. 1-3):
//   h1 = W1 k, h3 = W3 k, a = SiLU(h1), u = a ⊙ h3, du = -W2^T v
//   dh3 = du ⊙ a, dh1 = du ⊙ h3 ⊙ SiLU'(h1)
//   G1 = Σ η dh1 k^T, G3 = Σ η dh3 k^T, G2 = -Σ η v u^T

#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace ttt {
namespace {

constexpr int kT = 64;    // token (or query) tile
constexpr int kJ = 64;    // hidden tile
constexpr int kC = 16;    // contraction step

// ----------------------------------------------------------------------------
// Forward + backward elementwise: writes η·u, η·dh1, η·dh3 ([H][n][hid]).
// grid = (ceil(n/64), hid/64, H), 256 threads, 4x4 outputs per thread.
__global__ void __launch_bounds__(256) f32_fwd_bwd_kernel(
    const float* __restrict__ K, const float* __restrict__ V, const float* __restrict__ eta,
    const float* __restrict__ W1, const float* __restrict__ W2, const float* __restrict__ W3,
    int64_t n, int H, int d, int hid, float* __restrict__ U, float* __restrict__ DH1,
    float* __restrict__ DH3) {
  __shared__ float sK[kC][kT + 4], sV[kC][kT + 4];
  __shared__ float sW1[kC][kJ + 4], sW3[kC][kJ + 4], sW2[kC][kJ + 4];
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const int64_t t0 = (int64_t)blockIdx.x * kT;
  const int j0 = blockIdx.y * kJ, head = blockIdx.z;
  const int64_t ld = (int64_t)H * d;
  const float* w1 = W1 + (size_t)head * hid * d;
  const float* w3 = W3 + (size_t)head * hid * d;
  const float* w2 = W2 + (size_t)head * d * hid;
  float a1[4][4] = {}, a3[4][4] = {}, a2[4][4] = {};
  for (int c0 = 0; c0 < d; c0 += kC) {
    for (int e = tid; e < kT * kC; e += 256) {
      const int t = e / kC, c = e % kC;
      const int64_t tok = t0 + t;
      float kv = 0.f, vv = 0.f;
      if (tok < n) {
        kv = K[tok * ld + (int64_t)head * d + c0 + c];
        vv = V[tok * ld + (int64_t)head * d + c0 + c];
      }
      sK[c][t] = kv;
      sV[c][t] = vv;
      const int j = e / kC;
      sW1[c][j] = w1[(size_t)(j0 + j) * d + c0 + c];
      sW3[c][j] = w3[(size_t)(j0 + j) * d + c0 + c];
      const int c2 = e / kJ, j2 = e % kJ;
      sW2[c2][j2] = w2[(size_t)(c0 + c2) * hid + j0 + j2];
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < kC; ++c) {
      float k4[4], v4[4], p1[4], p3[4], p2[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        k4[i] = sK[c][ty * 4 + i];
        v4[i] = sV[c][ty * 4 + i];
        p1[i] = sW1[c][tx * 4 + i];
        p3[i] = sW3[c][tx * 4 + i];
        p2[i] = sW2[c][tx * 4 + i];
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          a1[a][b] = fmaf(k4[a], p1[b], a1[a][b]);
          a3[a][b] = fmaf(k4[a], p3[b], a3[a][b]);
          a2[a][b] = fmaf(v4[a], p2[b], a2[a][b]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int64_t tok = t0 + ty * 4 + a;
    if (tok >= n) continue;
    const float e = eta[tok * H + head];
    float ou[4], o1[4], o3[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const float h1 = a1[a][b], h3 = a3[a][b], du = -a2[a][b];
      const float s = 1.f / (1.f + expf(-h1));
      const float act = h1 * s;
      ou[b] = e * (act * h3);
      o3[b] = e * (du * act);
      o1[b] = e * (du * h3 * (s * (1.f + h1 * (1.f - s))));
    }
    const size_t off = ((size_t)head * n + tok) * hid + j0 + tx * 4;
    *reinterpret_cast<float4*>(U + off) = make_float4(ou[0], ou[1], ou[2], ou[3]);
    *reinterpret_cast<float4*>(DH1 + off) = make_float4(o1[0], o1[1], o1[2], o1[3]);
    *reinterpret_cast<float4*>(DH3 + off) = make_float4(o3[0], o3[1], o3[2], o3[3]);
  }
}

// ----------------------------------------------------------------------------
// Token reduction, split-K.  Partial s of matrix m for one head:
//   m=0: P1[j][c] = Σ_t DH1[t][j] K[t][c]     m=1: P3 likewise with DH3
//   m=2: P2[c][j] = Σ_t U[t][j] V[t][c]       (= -G2)
// Each split s sums tokens [s*chunk, min(n,(s+1)*chunk)) in increasing order.
// grid = ((hid/64)*(d/64), 3*H, S), 256 threads.
__global__ void __launch_bounds__(256) f32_grad_kernel(
    const float* __restrict__ U, const float* __restrict__ DH1, const float* __restrict__ DH3,
    const float* __restrict__ K, const float* __restrict__ V, int64_t n, int H, int d, int hid,
    int64_t chunk, float* __restrict__ partials) {
  __shared__ float sA[kC][kJ + 4], sB[kC][kJ + 4];
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const int jt = blockIdx.x % (hid / kJ), ct = blockIdx.x / (hid / kJ);
  const int j0 = jt * kJ, c0 = ct * kJ;
  const int m = blockIdx.y % 3, head = blockIdx.y / 3, s = blockIdx.z;
  const float* A = (m == 0 ? DH1 : m == 1 ? DH3 : U) + (size_t)head * n * hid;
  const float* B = (m == 2 ? V : K);
  const int64_t ld = (int64_t)H * d;
  const int64_t ts = (int64_t)s * chunk;
  const int64_t te = ts + chunk < n ? ts + chunk : n;
  float acc[4][4] = {};
  for (int64_t t0 = ts; t0 < te; t0 += kC) {
    for (int e = tid; e < kC * kJ; e += 256) {
      const int t = e / kJ, x = e % kJ;
      const int64_t tok = t0 + t;
      float av = 0.f, bv = 0.f;
      if (tok < te) {
        av = A[tok * hid + j0 + x];
        bv = B[tok * ld + (int64_t)head * d + c0 + x];
      }
      sA[t][x] = av;
      sB[t][x] = bv;
    }
    __syncthreads();
#pragma unroll
    for (int t = 0; t < kC; ++t) {
      float a4[4], b4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a4[i] = sA[t][ty * 4 + i];
        b4[i] = sB[t][tx * 4 + i];
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(a4[a], b4[b], acc[a][b]);
    }
    __syncthreads();
  }
  float* P = partials + (((size_t)s * H + head) * 3 + m) * (size_t)hid * d;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = j0 + ty * 4 + a, c = c0 + tx * 4 + b;
      if (m < 2)
        P[(size_t)j * d + c] = acc[a][b];
      else
        P[(size_t)c * hid + j] = acc[a][b];
    }
}

// ----------------------------------------------------------------------------
// Apply: O = W2 [SiLU(W1 q) ⊙ W3 q] for 32 queries of one head per block.
// The hidden activations of the block stay in shared memory.
constexpr int kQ = 32;
__global__ void __launch_bounds__(256) f32_apply_kernel(
    const float* __restrict__ Q, const float* __restrict__ W1, const float* __restrict__ W2,
    const float* __restrict__ W3, int64_t m, int H, int d, int hid, float* __restrict__ O) {
  extern __shared__ float sU[];  // [kQ][hid]
  __shared__ float sQ[kC][kQ + 4], sW1[kC][kJ + 4], sW3[kC][kJ + 4];
  __shared__ float sW2[kC][kJ + 4];
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const int64_t q0 = (int64_t)blockIdx.x * kQ;
  const int head = blockIdx.y;
  const int64_t ld = (int64_t)H * d;
  const float* w1 = W1 + (size_t)head * hid * d;
  const float* w3 = W3 + (size_t)head * hid * d;
  const float* w2 = W2 + (size_t)head * d * hid;
  for (int j0 = 0; j0 < hid; j0 += kJ) {
    float a1[2][4] = {}, a3[2][4] = {};
    for (int c0 = 0; c0 < d; c0 += kC) {
      for (int e = tid; e < kQ * kC; e += 256) {
        const int q = e / kC, c = e % kC;
        const int64_t qi = q0 + q;
        sQ[c][q] = qi < m ? Q[qi * ld + (int64_t)head * d + c0 + c] : 0.f;
      }
      for (int e = tid; e < kJ * kC; e += 256) {
        const int j = e / kC, c = e % kC;
        sW1[c][j] = w1[(size_t)(j0 + j) * d + c0 + c];
        sW3[c][j] = w3[(size_t)(j0 + j) * d + c0 + c];
      }
      __syncthreads();
#pragma unroll
      for (int c = 0; c < kC; ++c) {
        const float qa = sQ[c][ty * 2], qb = sQ[c][ty * 2 + 1];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const float p1 = sW1[c][tx * 4 + b], p3 = sW3[c][tx * 4 + b];
          a1[0][b] = fmaf(qa, p1, a1[0][b]);
          a1[1][b] = fmaf(qb, p1, a1[1][b]);
          a3[0][b] = fmaf(qa, p3, a3[0][b]);
          a3[1][b] = fmaf(qb, p3, a3[1][b]);
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const float h1 = a1[a][b];
        const float s = 1.f / (1.f + expf(-h1));
        sU[(ty * 2 + a) * hid + j0 + tx * 4 + b] = h1 * s * a3[a][b];
      }
  }
  __syncthreads();
  for (int c0 = 0; c0 < d; c0 += kJ) {
    float acc[2][4] = {};
    for (int j0 = 0; j0 < hid; j0 += kC) {
      for (int e = tid; e < kJ * kC; e += 256) {
        const int c = e / kC, j = e % kC;
        sW2[j][c] = w2[(size_t)(c0 + c) * hid + j0 + j];
      }
      __syncthreads();
#pragma unroll
      for (int j = 0; j < kC; ++j) {
        const float ua = sU[(ty * 2) * hid + j0 + j], ub = sU[(ty * 2 + 1) * hid + j0 + j];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const float w = sW2[j][tx * 4 + b];
          acc[0][b] = fmaf(ua, w, acc[0][b]);
          acc[1][b] = fmaf(ub, w, acc[1][b]);
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 2; ++a) {
      const int64_t qi = q0 + ty * 2 + a;
      if (qi >= m) continue;
      float* o = O + qi * ld + (int64_t)head * d + c0 + tx * 4;
      *reinterpret_cast<float4*>(o) = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
    }
  }
}

// Gated output unit, fp32: block (16 rows, head); o' rows staged in shared
// memory, one thread per output column j computes g_j = W_g[j,:] o' for the
// 16 rows, the RMS is formed in fp64 per row.
constexpr int kGR = 16;
__global__ void __launch_bounds__(256) f32_gate_kernel(const float* __restrict__ Wg,
                                                       const float* Oin, float* Oout, int64_t m,
                                                       int H, int d, float eps) {
  __shared__ float so[kGR][256];
  __shared__ float inv[kGR];
  const int head = blockIdx.y;
  const int64_t r0 = (int64_t)blockIdx.x * kGR;
  const size_t ld = (size_t)H * d;
  for (int i = threadIdx.x; i < kGR * d; i += blockDim.x) {
    const int t = i / d, c = i % d;
    so[t][c] = r0 + t < m ? Oin[(size_t)(r0 + t) * ld + (size_t)head * d + c] : 0.f;
  }
  __syncthreads();
  if (threadIdx.x < kGR) {
    double ss = 0.0;
    for (int c = 0; c < d; ++c) ss += (double)so[threadIdx.x][c] * so[threadIdx.x][c];
    inv[threadIdx.x] = (float)(1.0 / sqrt(ss / d + (double)eps));
  }
  __syncthreads();
  const float* W = Wg + (size_t)head * d * d;
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    float acc[kGR];
#pragma unroll
    for (int t = 0; t < kGR; ++t) acc[t] = 0.f;
    for (int k = 0; k < d; ++k) {
      const float w = W[(size_t)j * d + k];
#pragma unroll
      for (int t = 0; t < kGR; ++t) acc[t] = fmaf(w, so[t][k], acc[t]);
    }
#pragma unroll
    for (int t = 0; t < kGR; ++t)
      if (r0 + t < m)
        Oout[(size_t)(r0 + t) * ld + (size_t)head * d + j] =
            so[t][j] * inv[t] * (acc[t] / (1.f + expf(-acc[t])));
  }
}

}  // namespace

SplitPlan f32_split_plan(const Problem& p) {
  const int tiles = (p.hid / kJ) * (p.d / kJ) * 3 * p.H;
  int S = (2 * 148 + tiles - 1) / tiles;
  const int64_t max_s = (p.n + 255) / 256;
  if (S > max_s) S = (int)(max_s < 1 ? 1 : max_s);
  int64_t chunk = (p.n + S - 1) / S;
  chunk = (chunk + kC - 1) / kC * kC;
  if (chunk < kC) chunk = kC;
  return {S, chunk};
}

// Bytes of the update's own workspace; the optional Newton-Schulz region
// follows it at a 1024-byte boundary.
static size_t f32_main_bytes(const Problem& p) {
  const SplitPlan sp = f32_split_plan(p);
  size_t b = 0;
  b += align_up(3 * (size_t)p.H * p.n * p.hid * sizeof(float), 256);
  b += align_up((size_t)sp.S * p.H * 3 * p.hid * p.d * sizeof(float), 256);
  b += align_up((size_t)p.H * (2 * p.hid + p.d) * 2 * sizeof(double), 256);
  return align_up(b, 1024);
}

size_t f32_workspace_bytes(const Problem& p) { return f32_main_bytes(p) + ns_workspace_bytes(p); }

cudaError_t f32_update(const Problem& p, const float* W1, const float* W2, const float* W3,
                       const float* K, const float* V, const float* eta, float* W1o, float* W2o,
                       float* W3o, __nv_bfloat16_raw* shadow, void* ws, cudaStream_t st,
                       float* partial_out) {
  const SplitPlan sp = f32_split_plan(p);
  char* w = static_cast<char*>(ws);
  const size_t inter = (size_t)p.H * p.n * p.hid;
  float* U = reinterpret_cast<float*>(w);
  float* DH1 = U + inter;
  float* DH3 = DH1 + inter;
  w += align_up(3 * inter * sizeof(float), 256);
  float* partials = reinterpret_cast<float*>(w);
  w += align_up((size_t)sp.S * p.H * 3 * p.hid * p.d * sizeof(float), 256);
  float* scratch = reinterpret_cast<float*>(w);
  if (p.n > 0) {
    dim3 g1((unsigned)((p.n + kT - 1) / kT), p.hid / kJ, p.H);
    {
      TraceScope ts("f32_fwd_bwd", st);
      f32_fwd_bwd_kernel<<<g1, 256, 0, st>>>(K, V, eta, W1, W2, W3, p.n, p.H, p.d, p.hid, U, DH1,
                                            DH3);
    }
    dim3 g2((p.hid / kJ) * (p.d / kJ), 3 * p.H, sp.S);
    {
      TraceScope ts("f32_grad", st);
      f32_grad_kernel<<<g2, 256, 0, st>>>(U, DH1, DH3, K, V, p.n, p.H, p.d, p.hid, sp.chunk,
                                         partials);
    }
  } else {
    const cudaError_t m =
        cudaMemsetAsync(partials, 0, (size_t)sp.S * p.H * 3 * p.hid * p.d * sizeof(float), st);
    if (m != cudaSuccess) return m;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (partial_out != nullptr)
    return sum_splits(sp.S, (size_t)p.H * 3 * p.hid * p.d, partials, partial_out, st);
  return ns_then_renorm(p, sp.S, partials, static_cast<char*>(ws) + f32_main_bytes(p), false, W1,
                        W2, W3, W1o, W2o, W3o, shadow, scratch, st);
}

cudaError_t f32_apply(const Problem& p, const float* W1, const float* W2, const float* W3,
                      const float* Q, float* O, cudaStream_t st) {
  if (p.n == 0) return cudaSuccess;
  const size_t smem = (size_t)kQ * p.hid * sizeof(float);
  // The limit is raised once, to what the largest supported hidden width needs.
  cudaError_t e = ensure_smem_attr(f32_apply_kernel, (int)(kQ * 512 * sizeof(float)));
  if (e != cudaSuccess) return e;
  dim3 g((unsigned)((p.n + kQ - 1) / kQ), p.H);
  TraceScope ts("f32_apply", st);
  f32_apply_kernel<<<g, 256, smem, st>>>(Q, W1, W2, W3, p.n, p.H, p.d, p.hid, O);
  return cudaGetLastError();
}

cudaError_t f32_gate(const Problem& p, const float* Wg, const float* Oin, float* Oout, float eps,
                     cudaStream_t st) {
  if (p.n == 0) return cudaSuccess;
  dim3 g((unsigned)((p.n + kGR - 1) / kGR), p.H);
  TraceScope ts("f32_gate", st);
  f32_gate_kernel<<<g, 256, 0, st>>>(Wg, Oin, Oout, p.n, p.H, p.d, eps);
  return cudaGetLastError();
}

}  // namespace ttt
