// Newton-Schulz orthonormalisation of the fast-weight gradient (ZipMap review,
// section 2 "Feature Backbone", the update after Eq. 3: Delta <- NewtonSchulz(g)
// "following the Muon optimizer"; the L2 renormalisation then acts on
// W - Delta).  The pages give neither the polynomial nor the step count; the
// iteration is Muon's published quintic (Jordan et al. 2024):
//
//   X0 = g / ||g||_F,   X <- a X + (b A + c A^2) X,   A = X X^T,
//   (a, b, c) = (3.4445, -4.7750, 2.0315),
//
// on the wide orientation of each matrix.  Per head, g1 and g3 ([hidden][d])
// are worked as their transposes and g2 ([d][hidden]) as is, so every matrix
// is d x hidden ("working layout", rows padded with zeros to a multiple of
// 128: padded rows stay zero through the iteration).
//
// Stages (all on the caller's stream):
//   ns_gather   sum the split-K partials in fixed order, transpose into the
//               working layout, per-32x32-tile sums of squares (fp64)
//   ns_scale    fixed-order Frobenius norm, X0 = G / ||G||_F in fp32 and as
//               its bf16 pair (hi, lo), zero padding
//   iterations  tensor cores: one clustered tcgen05 kernel for all steps;
//               check mode: three fp32 CUDA-core GEMMs per step
//   ns_finish   Delta back to the partials layout (S = 1) for reduce_renorm
//
// Tensor-core precision: a bf16 MMA of plain operands loses too much through
// five quintic steps, so every operand x is split as hi = bf16(x),
// lo = bf16(x - hi) and each product is hi*hi + hi*lo + lo*hi with fp32
// accumulation in TMEM; each CTA keeps its own tiles of the iterate (and of
// A between phases) in fp32 in TMEM, so only the bf16 pairs travel.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "tc_util.cuh"

namespace ttt {
namespace {

constexpr float kNsA = 3.4445f, kNsB = -4.7750f, kNsC = 2.0315f;

// Rows of the working layout: d rounded up to a multiple of 128.
__host__ __device__ inline int ns_rows(int d) { return (d + 127) / 128 * 128; }

// ----------------------------------------------------------------------------
// Gather: one block per (head, matrix, 32 x 32 tile of the d x hidden working
// matrix).  Partials layout [S][H][3][hid*d]: block 0 = G1 [hid][d], block 1 =
// G3 [hid][d], block 2 = -G2 [d][hid].  Working matrix index m = head*3 + blk.
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256) ns_gather_kernel(const float* __restrict__ partials, int S,
                                                        int H, int d, int hid, int Rp,
                                                        float* __restrict__ X,
                                                        double* __restrict__ tile_ss) {
  __shared__ float tile[32][33];
  __shared__ double red[8];
  const int tiles_c = d / 32, tiles_j = hid / 32, per = tiles_c * tiles_j;
  const int m = blockIdx.x / per, t = blockIdx.x % per;
  const int head = m / 3, blk = m % 3;
  const int c0 = (t / tiles_j) * 32, j0 = (t % tiles_j) * 32;  // working rows c, cols j
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const size_t mat = (size_t)hid * d;
  // blocks 0/1: read G rows j (coalesced along c); block 2: read rows c
  // (coalesced along j).  tile[a][b] holds working element (c0+b, j0+a) for
  // blocks 0/1 and (c0+a, j0+b) for block 2.  Each thread owns 4 elements
  // (rows ty, ty+8, ...) and sums them over s in increasing order.
  size_t off[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty + 8 * i;
    off[i] = blk < 2 ? (size_t)(j0 + r) * d + c0 + tx : (size_t)(c0 + r) * hid + j0 + tx;
  }
  const size_t sstride = (size_t)H * 3 * mat;
  const float* P = partials + ((size_t)head * 3 + blk) * mat;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  int s = 0;
  for (; s + 2 <= S; s += 2) {  // two splits' loads in flight, added in split order
    float a[4], b[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      a[i] = P[(size_t)s * sstride + off[i]];
      b[i] = P[(size_t)(s + 1) * sstride + off[i]];
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = (acc[i] + (double)a[i]) + (double)b[i];
  }
  if (s < S) {
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] += (double)P[(size_t)s * sstride + off[i]];
  }
  double ss = 0.0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float v = blk < 2 ? (float)acc[i] : (float)(-acc[i]);
    tile[ty + 8 * i][tx] = v;
    ss = fma((double)v, (double)v, ss);
  }
  __syncthreads();
  float* Xm = X + (size_t)m * Rp * hid;
  for (int r = ty; r < 32; r += 8) {
    const float v = blk < 2 ? tile[tx][r] : tile[r][tx];
    Xm[(size_t)(c0 + r) * hid + j0 + tx] = v;
  }
  // fixed-order block sum of the squares
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (tx == 0) red[ty] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int i = 0; i < 8; ++i) s += red[i];
    tile_ss[blockIdx.x] = s;
  }
}

// Scale: grid (matrix, slice of rows).  Every block forms the same
// fixed-order norm from the tile sums, scales its rows by 1/||G||_F (zero
// gradient -> zero) and clears the padding rows.
__global__ void __launch_bounds__(256) ns_scale_kernel(int d, int hid, int Rp, int tiles,
                                                       const double* __restrict__ tile_ss,
                                                       float* __restrict__ X,
                                                       __nv_bfloat16* __restrict__ Xh,
                                                       __nv_bfloat16* __restrict__ Xl) {
  __shared__ double inv;
  const int m = blockIdx.y;
  if (threadIdx.x < 32) {
    // lane l sums tiles l, l+32, ... in order; then a fixed butterfly
    double s = 0.0;
    for (int i = threadIdx.x; i < tiles; i += 32) s += tile_ss[(size_t)m * tiles + i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) inv = s > 0.0 ? 1.0 / sqrt(s) : 0.0;
  }
  __syncthreads();
  const int rows_per = Rp / gridDim.x;
  const int q_per_row = hid / 4;  // 4 columns per thread step
  const size_t mo = (size_t)m * Rp * hid;
  for (int i = threadIdx.x; i < rows_per * q_per_row; i += blockDim.x) {
    const int row = blockIdx.x * rows_per + i / q_per_row, col = 4 * (i % q_per_row);
    const size_t o = mo + (size_t)row * hid + col;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row < d) {
      const float4 x = *reinterpret_cast<const float4*>(X + o);
      v = make_float4((float)((double)x.x * inv), (float)((double)x.y * inv),
                      (float)((double)x.z * inv), (float)((double)x.w * inv));
    }
    *reinterpret_cast<float4*>(X + o) = v;
    // the bf16 pair the tensor-core iteration reads: hi + lo carries ~16 bits
    const float f[4] = {v.x, v.y, v.z, v.w};
    uint32_t hp[2], lp[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const __nv_bfloat16 h0 = __float2bfloat16_rn(f[2 * k]), h1 = __float2bfloat16_rn(f[2 * k + 1]);
      hp[k] = pack_bf16x2(__bfloat162float(h0), __bfloat162float(h1));
      lp[k] = pack_bf16x2(f[2 * k] - __bfloat162float(h0), f[2 * k + 1] - __bfloat162float(h1));
    }
    *reinterpret_cast<uint2*>(Xh + o) = make_uint2(hp[0], hp[1]);
    *reinterpret_cast<uint2*>(Xl + o) = make_uint2(lp[0], lp[1]);
  }
}

// Finish: Delta (working layout) back to the partials layout of one split:
// blocks 0/1 transposed to [hid][d], block 2 negated (reduce_renorm adds
// block 2 and subtracts blocks 0/1, so every matrix becomes W - Delta).
__global__ void __launch_bounds__(256) ns_finish_kernel(const float* __restrict__ X, int H, int d,
                                                        int hid, int Rp,
                                                        float* __restrict__ delta) {
  __shared__ float tile[32][33];
  const int tiles_c = d / 32, tiles_j = hid / 32, per = tiles_c * tiles_j;
  const int m = blockIdx.x / per, t = blockIdx.x % per;
  const int blk = m % 3;
  const int c0 = (t / tiles_j) * 32, j0 = (t % tiles_j) * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const float* Xm = X + (size_t)m * Rp * hid;
  float* Dm = delta + (size_t)m * hid * d;  // [H][3] blocks are consecutive
  if (blk == 2) {
    for (int r = ty; r < 32; r += 8) {
      const size_t off = (size_t)(c0 + r) * hid + j0 + tx;
      Dm[off] = -Xm[off];
    }
    return;
  }
  for (int r = ty; r < 32; r += 8) tile[r][tx] = Xm[(size_t)(c0 + r) * hid + j0 + tx];
  __syncthreads();
  for (int r = ty; r < 32; r += 8) Dm[(size_t)(j0 + r) * d + c0 + tx] = tile[tx][r];
}

// ----------------------------------------------------------------------------
// Check mode: batched fp32 GEMM on CUDA cores,
//   O[b] = alpha * P[b] op(Q[b]) + beta * R[b],
// op(Q) = Q^T (Q stored [N][K]) when QT, else Q ([K][N]).  64 x 64 tiles,
// 16-deep k steps, each thread 4 x 4 outputs; every dimension is a multiple
// of 64.  R (nullable) has O's pitch.
// ----------------------------------------------------------------------------
template <bool QT>
__global__ void __launch_bounds__(256) ns_f32_gemm_kernel(
    const float* __restrict__ P, const float* __restrict__ Q, const float* __restrict__ R,
    float* __restrict__ O, int K, int ldp, int ldq, int ldo, size_t sp, size_t sq, size_t so,
    float alpha, float beta) {
  __shared__ float sP[16][68];  // [k][i]
  __shared__ float sQ[16][68];  // [k][j]
  const size_t b = blockIdx.z;
  P += b * sp;
  Q += b * sq;
  O += b * so;
  if (R != nullptr) R += b * so;
  const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int e = threadIdx.x; e < 1024; e += 256) {
      const int i = e >> 4, k = e & 15;
      sP[k][i] = P[(size_t)(i0 + i) * ldp + k0 + k];
      if (QT) {
        sQ[k][i] = Q[(size_t)(j0 + i) * ldq + k0 + k];
      } else {
        const int kk = e >> 6, j = e & 63;
        sQ[kk][j] = Q[(size_t)(k0 + kk) * ldq + j0 + j];
      }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float a[4], q[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        a[r] = sP[k][ty * 4 + r];
        q[r] = sQ[k][tx * 4 + r];
      }
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(a[r], q[c], acc[r][c]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const size_t row = (size_t)(i0 + ty * 4 + r) * ldo;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int col = j0 + tx * 4 + c;
      float v = alpha * acc[r][c];
      if (R != nullptr) v = fmaf(beta, R[row + col], v);
      O[row + col] = v;
    }
  }
}

// ----------------------------------------------------------------------------
// Tensor-core iteration.  One cluster of (Rp/128)^2 CTAs per working matrix
// runs every step.  Each GEMM's epilogue writes its result as a bf16 pair
// hi = bf16(x), lo = bf16(x - hi) (TMA bulk stores; the fp32 value stays in
// TMEM where a later epilogue of the same CTA needs it);
// the next GEMM's operands are those pairs, loaded by TMA (128-byte swizzle)
// into a two-stage ring, and each product is hi*hi + hi*lo + lo*hi with fp32
// accumulation in TMEM.  Per CTA (cluster rank r, mi = r / RB, ni = r % RB,
// RB = Rp / 128):
//   phase 0  A  = X X^T        tile rows mi*128, cols ni*128  (K = hidden)
//   phase 1  B  = b A + c A A  same tile                      (K = Rp; A is
//                              symmetric, so rows of A serve as B operand)
//   phase 2  X' = a X + B X    rows mi*128, cols ni*N3        (K = Rp, X as
//                              MN-major B operand)
// The cluster meets at a hardware barrier (release/acquire) after every
// phase; the epilogues' generic stores are fenced against the next phase's
// TMA loads on both sides of that barrier.  Warps: 0 TMA producer (one
// thread), 1 MMA issuer (one thread), 2..9 epilogue (two per TMEM lane
// quadrant, each half of the tile's columns).
// ----------------------------------------------------------------------------
template <int RP, int C>
struct NSL {
  static constexpr int RB = RP / 128;
  static constexpr int CL = RB * RB;        // CTAs per cluster
  static constexpr int N3 = C / RB;         // width of the X' tile
  static constexpr int A_T = 128 * 128;     // 128 rows x 64 bf16 = 16 KB
  static constexpr int B_T = N3 * 128;      // widest B tile of one k chunk
  static constexpr int STAGE = 2 * A_T + 2 * B_T;
  static constexpr int NST = 2;
  static constexpr int OFF_BAR = NST * STAGE;
  static constexpr int SMEM = OFF_BAR + 64 + 1024;  // + alignment slack
  static constexpr int TMEM = 512;  // accumulator, A tile, X tile (see kAR, kXR)
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static_assert(N3 % 64 == 0 && N3 <= 256, "X' tile width");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

// Tensor maps of the iterates (bf16, 128-byte swizzle, 64-element inner box).
struct NsMaps {
  CUtensorMap xh[2], xl[2];    // X hi / lo, K-major view: box {64 k, 128 rows}
  CUtensorMap xhm[2], xlm[2];  // X hi / lo, MN-major view: box {64 cols, 64 k rows,
                               // N3/64 column blocks}, landing as [block][row][128 B]
  CUtensorMap ah, al, bh, bl;  // A, B hi / lo, K-major: box {64 k, 128 rows}
};
// fp32 iterates of all matrices (matrix m at m * Rp * C).
struct NsBufs {
  float* xf[2];  // fp32 iterates: X0 (read at start), the final X (written on the last step)
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Every thread of every CTA of the cluster; global writes before it are
// visible to the cluster's reads after it.
__device__ __forceinline__ void cluster_barrier() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

template <int CL>
__device__ __forceinline__ void ns_sync() {
  if (CL > 1)
    cluster_barrier();
  else
    __syncthreads();
}

// TMEM columns: [0, N) the accumulator; [kAR, kAR + 128) this CTA's A tile
// in fp32, from phase 0's epilogue to phase 1's (phase 0/1 accumulators use
// only [0, 128)); [kXR, kXR + N3) this CTA's X tile in fp32, kept across
// steps (phase 2 reads it and writes X' back).  So no epilogue reads fp32
// operands from global memory.
constexpr uint32_t kAR = 128, kXR = 256, kNsTmemCols = 512;

// Epilogue of one 128 x N tile: warp w reads TMEM lanes 32*(w%4).. (its rows)
// and half (w-2)/4 of the columns.  MODE 0: x = acc, kept in TMEM for phase
// 1; MODE 1: x = b A + c acc (A from TMEM); MODE 2: x = a X + acc (X from
// TMEM, x written back; on the last step also stored in fp32 to xf_out).
// hi/lo of x are staged in the (idle) ring as 128-byte-swizzled [128 x 64]
// chunks and written with TMA bulk stores through maps mh / ml at column x0,
// row y0; the stores have completed when the function returns.
template <int N, int MODE>
__device__ __forceinline__ void ns_epilogue(uint64_t* acc_full, uint32_t parity, uint32_t tmem,
                                            uint8_t* stage, const CUtensorMap* mh,
                                            const CUtensorMap* ml, int x0, int y0,
                                            float* xf_out, int ldf, volatile int* abort,
                                            int* err) {
  constexpr int HALF = N / 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3, half = (warp - 2) >> 2;
  const int row = 32 * q + lane;
  const uint32_t lanes = (uint32_t)(32 * q) << 16;
  TTT_DCHECK(kXR + N <= kNsTmemCols && HALF % 32 == 0, err, kErrCheckTmem);
  uint8_t* hi = stage;
  uint8_t* lo = stage + N * 256;  // N/64 chunks of 16 KB
  mbar_wait(acc_full, parity, abort, err, kErrWaitAcc);
  tc_fence_after();
#pragma unroll 1
  for (int j = 0; j < HALF / 32; ++j) {
    const int col = half * HALF + 32 * j;
    uint32_t v[32];
    tmem_ld_32x32(tmem + lanes + (uint32_t)col, v);
    uint32_t rr[32];
    if constexpr (MODE == 1) tmem_ld_32x32(tmem + lanes + kAR + (uint32_t)col, rr);
    if constexpr (MODE == 2) tmem_ld_32x32(tmem + lanes + kXR + (uint32_t)col, rr);
    tmem_ld_wait();
    uint32_t xb[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const float acc = __uint_as_float(v[e]);
      float x = acc;
      if constexpr (MODE == 1) x = fmaf(kNsC, acc, kNsB * __uint_as_float(rr[e]));
      if constexpr (MODE == 2) x = fmaf(kNsA, __uint_as_float(rr[e]), acc);
      xb[e] = __float_as_uint(x);
    }
    if constexpr (MODE == 0) tmem_st_32x32(tmem + lanes + kAR + (uint32_t)col, xb);
    if constexpr (MODE == 2) {
      tmem_st_32x32(tmem + lanes + kXR + (uint32_t)col, xb);
      if (xf_out != nullptr) {
        float* o = xf_out + (size_t)row * ldf + col;
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          __stcg(reinterpret_cast<float4*>(o + e),
                 make_float4(__uint_as_float(xb[e]), __uint_as_float(xb[e + 1]),
                             __uint_as_float(xb[e + 2]), __uint_as_float(xb[e + 3])));
      }
    }
    uint32_t h[16], l[16];
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const float x0f = __uint_as_float(xb[e]), x1f = __uint_as_float(xb[e + 1]);
      const __nv_bfloat16 a0 = __float2bfloat16_rn(x0f), a1 = __float2bfloat16_rn(x1f);
      h[e / 2] = pack_bf16x2(__bfloat162float(a0), __bfloat162float(a1));
      l[e / 2] = pack_bf16x2(x0f - __bfloat162float(a0), x1f - __bfloat162float(a1));
    }
    // 32 columns = 4 16-byte units of one 64-column chunk
    const int chunk = col / 64, u0 = (col % 64) / 8;
    const int base = chunk * 16384 + row * 128;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int off = base + (((u0 + e) ^ (row & 7)) << 4);
      *reinterpret_cast<uint4*>(hi + off) = make_uint4(h[4 * e], h[4 * e + 1], h[4 * e + 2], h[4 * e + 3]);
      *reinterpret_cast<uint4*>(lo + off) = make_uint4(l[4 * e], l[4 * e + 1], l[4 * e + 2], l[4 * e + 3]);
    }
  }
  if constexpr (MODE != 1) tmem_st_wait();
  tc_fence_before();
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  named_bar_sync(5, 32 * (NSL<256, 512>::EPI_WARPS));
  if (warp == 2 && lane == 0) {
    for (int c = 0; c < N / 64; ++c) {
      tma_store_2d(mh, hi + c * 16384, x0 + 64 * c, y0);
      tma_store_2d(ml, lo + c * 16384, x0 + 64 * c, y0);
    }
    bulk_commit_group();
    bulk_wait_group0();
    fence_proxy_async_global();
  }
}

template <int RP, int C>
__global__ void __launch_bounds__(NSL<RP, C>::THREADS, 1)
    ns_tc_kernel(const __grid_constant__ NsMaps maps, const NsBufs buf, int steps, int* err) {
  using L = NSL<RP, C>;
  extern __shared__ uint8_t ns_raw[];
  uint8_t* smem = align1024(ns_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* empty = full + 2;
  uint64_t* acc_full = empty + 2;
  uint64_t* done = acc_full + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = L::CL > 1 ? (int)cluster_rank() : 0;
  const int m = blockIdx.x / L::CL;
  const int mi = rank / L::RB, ni = rank % L::RB;
  const int mrow = m * RP;  // first row of this matrix in the stacked views
  const size_t xo = (size_t)m * RP * C, ao = (size_t)m * RP * RP;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tslot, L::TMEM);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  if (warp >= 2) {
    // this CTA's X tile (rows mi*128.., cols ni*N3..) into TMEM, fp32
    const int q = warp & 3, half = (warp - 2) >> 2;
    const float* xr = buf.xf[0] + xo + (size_t)(mi * 128 + 32 * q + lane) * C + ni * L::N3;
#pragma unroll 1
    for (int j = 0; j < L::N3 / 64; ++j) {
      const int col = half * (L::N3 / 2) + 32 * j;
      uint32_t xb[32];
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const float4 f = __ldcg(reinterpret_cast<const float4*>(xr + col + e));
        xb[e] = __float_as_uint(f.x);
        xb[e + 1] = __float_as_uint(f.y);
        xb[e + 2] = __float_as_uint(f.z);
        xb[e + 3] = __float_as_uint(f.w);
      }
      tmem_st_32x32(tmem + ((uint32_t)(32 * q) << 16) + kXR + (uint32_t)col, xb);
    }
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  int g = 0;   // k chunks so far: ring slot g & 1, its (g >> 1)-th use
  int ph = 0;  // phases so far: parity of acc_full
  for (int it = 0; it < steps; ++it) {
    const int cur = it & 1, nxt = cur ^ 1;
    for (int p = 0; p < 3; ++p, ++ph) {
      const int nchunks = p == 0 ? C / 64 : RP / 64;
      if (warp == 0) {
        if (lane == 0) {
          // ------------------------------------------------ TMA producer
          fence_proxy_async_global();
          for (int j = 0; j < nchunks; ++j) {
            const int gj = g + j, s = gj & 1;
            if (gj >= 2) mbar_wait(&empty[s], ((gj >> 1) - 1) & 1, abort_flag, err, kErrWaitEmpty);
            uint8_t* st = smem + s * L::STAGE;
            uint8_t* bst = st + 2 * L::A_T;
            const int k0 = j * 64;
            TTT_DCHECK(mi * 128 + 128 <= RP && ni * 128 + 128 <= RP && k0 + 64 <= (p == 0 ? C : RP),
                       err, kErrCheckTma);
            if (p == 0) {
              mbar_arrive_expect_tx(&full[s], 4 * L::A_T);
              tma_load_2d(st, &maps.xh[cur], &full[s], k0, mrow + mi * 128);
              tma_load_2d(st + L::A_T, &maps.xl[cur], &full[s], k0, mrow + mi * 128);
              tma_load_2d(bst, &maps.xh[cur], &full[s], k0, mrow + ni * 128);
              tma_load_2d(bst + L::B_T, &maps.xl[cur], &full[s], k0, mrow + ni * 128);
            } else if (p == 1) {
              mbar_arrive_expect_tx(&full[s], 4 * L::A_T);
              tma_load_2d(st, &maps.ah, &full[s], k0, mrow + mi * 128);
              tma_load_2d(st + L::A_T, &maps.al, &full[s], k0, mrow + mi * 128);
              tma_load_2d(bst, &maps.ah, &full[s], k0, mrow + ni * 128);
              tma_load_2d(bst + L::B_T, &maps.al, &full[s], k0, mrow + ni * 128);
            } else {
              mbar_arrive_expect_tx(&full[s], 2 * L::A_T + 2 * L::B_T);
              tma_load_2d(st, &maps.bh, &full[s], k0, mrow + mi * 128);
              tma_load_2d(st + L::A_T, &maps.bl, &full[s], k0, mrow + mi * 128);
              tma_load_3d(bst, &maps.xhm[cur], &full[s], 0, mrow + k0, ni * (L::N3 / 64));
              tma_load_3d(bst + L::B_T, &maps.xlm[cur], &full[s], 0, mrow + k0, ni * (L::N3 / 64));
            }
          }
        }
      } else if (warp == 1) {
        if (lane == 0) {
          // ------------------------------------------------ MMA issuer
          const uint32_t idesc = p == 2 ? idesc_bf16_f32(128, L::N3, false, true)
                                        : idesc_bf16_f32(128, 128, false, false);
          for (int j = 0; j < nchunks; ++j) {
            const int gj = g + j, s = gj & 1;
            mbar_wait(&full[s], (gj >> 1) & 1, abort_flag, err, kErrWaitFull);
            tc_fence_after();
            const uint32_t a = smem_u32(smem + s * L::STAGE), b = a + 2 * L::A_T;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ah = sdesc_sw128(a + kk * 32, 16, 1024);
              const uint64_t al = sdesc_sw128(a + L::A_T + kk * 32, 16, 1024);
              const uint64_t bh = p == 2 ? sdesc_sw128(b + kk * 2048, 8192, 1024)
                                         : sdesc_sw128(b + kk * 32, 16, 1024);
              const uint64_t bl = p == 2 ? sdesc_sw128(b + L::B_T + kk * 2048, 8192, 1024)
                                         : sdesc_sw128(b + L::B_T + kk * 32, 16, 1024);
              umma_bf16(tmem, ah, bh, idesc, (j | kk) != 0);
              umma_bf16(tmem, ah, bl, idesc, 1);
              umma_bf16(tmem, al, bh, idesc, 1);
            }
            umma_commit(&empty[s]);
          }
          umma_commit(acc_full);
        }
      } else {
        // ------------------------------------------------ epilogue
        const uint32_t par = (uint32_t)(ph & 1);
        const int y0 = mrow + mi * 128;
        if (p == 0)
          ns_epilogue<128, 0>(acc_full, par, tmem, smem, &maps.ah, &maps.al, ni * 128, y0,
                              nullptr, 0, abort_flag, err);
        else if (p == 1)
          ns_epilogue<128, 1>(acc_full, par, tmem, smem, &maps.bh, &maps.bl, ni * 128, y0,
                              nullptr, 0, abort_flag, err);
        else
          ns_epilogue<L::N3, 2>(acc_full, par, tmem, smem, &maps.xh[nxt], &maps.xl[nxt],
                                ni * L::N3, y0,
                                it == steps - 1 ? buf.xf[nxt] + xo + (size_t)mi * 128 * C +
                                                      ni * L::N3
                                                : nullptr,
                                C, abort_flag, err);
      }
      g += nchunks;
      __syncwarp();
      ns_sync<L::CL>();
    }
  }
  if (warp == 0 && lane == 0) drain_ring(full, 2, g, err);
  if (warp == 1 && lane == 0) {
    umma_commit(done);
    volatile int never = 0;
    mbar_wait(done, 0, &never, err, kErrWaitFinal);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, L::TMEM);
  }
}

struct NsWs {
  float *X[2], *A, *B, *delta;     // fp32 iterates and products (B: check mode)
  __nv_bfloat16 *Xh[2], *Xl[2], *Ah, *Al, *Bh, *Bl;  // bf16 pairs (tensor cores)
  double* tile_ss;
};

NsWs ns_carve(const Problem& p, void* ws) {
  const int Rp = ns_rows(p.d);
  const size_t M = 3 * (size_t)p.H;
  const size_t xs = M * Rp * p.hid, as = M * Rp * Rp;
  char* c = static_cast<char*>(ws);
  NsWs w;
  auto f32 = [&](size_t n) {
    float* r = reinterpret_cast<float*>(c);
    c += align_up(n * 4, 1024);
    return r;
  };
  auto b16 = [&](size_t n) {
    __nv_bfloat16* r = reinterpret_cast<__nv_bfloat16*>(c);
    c += align_up(n * 2, 1024);
    return r;
  };
  w.X[0] = f32(xs);
  w.X[1] = f32(xs);
  w.A = f32(as);
  w.B = f32(as);
  w.delta = f32(M * p.hid * p.d);
  w.Xh[0] = b16(xs);
  w.Xh[1] = b16(xs);
  w.Xl[0] = b16(xs);
  w.Xl[1] = b16(xs);
  w.Ah = b16(as);
  w.Al = b16(as);
  w.Bh = b16(as);
  w.Bl = b16(as);
  w.tile_ss = reinterpret_cast<double*>(c);
  return w;
}

template <int RP, int C>
cudaError_t launch_ns_tc(const Problem& p, const NsWs& w, int* err, cudaStream_t st) {
  using L = NSL<RP, C>;
  const uint64_t rows = (uint64_t)3 * p.H * RP;  // all matrices stacked
  NsMaps maps;
  for (int b = 0; b < 2; ++b) {
    const uint64_t dk[2] = {(uint64_t)C, rows}, sk[1] = {(uint64_t)C * 2};
    const uint32_t bk[2] = {64, 128};
    const uint64_t dm[3] = {64, rows, (uint64_t)C / 64}, sm[2] = {(uint64_t)C * 2, 128};
    const uint32_t bm[3] = {64, 64, (uint32_t)(L::N3 / 64)};
    if (!make_map(&maps.xh[b], w.Xh[b], 2, dk, sk, bk) ||
        !make_map(&maps.xl[b], w.Xl[b], 2, dk, sk, bk) ||
        !make_map(&maps.xhm[b], w.Xh[b], 3, dm, sm, bm) ||
        !make_map(&maps.xlm[b], w.Xl[b], 3, dm, sm, bm))
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t da[2] = {(uint64_t)RP, rows}, sa[1] = {(uint64_t)RP * 2};
    const uint32_t ba[2] = {64, 128};
    if (!make_map(&maps.ah, w.Ah, 2, da, sa, ba) || !make_map(&maps.al, w.Al, 2, da, sa, ba) ||
        !make_map(&maps.bh, w.Bh, 2, da, sa, ba) || !make_map(&maps.bl, w.Bl, 2, da, sa, ba))
      return cudaErrorInvalidValue;
  }
  NsBufs buf;
  for (int b = 0; b < 2; ++b) buf.xf[b] = w.X[b];
  cudaError_t e = ensure_smem_attr(ns_tc_kernel<RP, C>, L::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(3 * p.H * L::CL));
  cfg.blockDim = dim3(L::THREADS);
  cfg.dynamicSmemBytes = L::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = L::CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = L::CL > 1 ? 1 : 0;
  TraceScope ts("ns_tc_iterate", st);
  return cudaLaunchKernelEx(&cfg, ns_tc_kernel<RP, C>, maps, buf, p.ns_steps, err);
}

}  // namespace

size_t ns_workspace_bytes(const Problem& p) {
  if (p.ns_steps <= 0) return 0;
  const int Rp = ns_rows(p.d);
  const size_t M = 3 * (size_t)p.H;
  const size_t tiles = (size_t)(p.d / 32) * (p.hid / 32);
  const size_t xs = M * Rp * p.hid, as = M * Rp * Rp;
  return 2 * align_up(xs * 4, 1024) + 2 * align_up(as * 4, 1024) +
         align_up(M * p.hid * p.d * 4, 1024) + 4 * align_up(xs * 2, 1024) +
         4 * align_up(as * 2, 1024) + align_up(M * tiles * 8, 1024);
}

cudaError_t ns_then_renorm(const Problem& p, int S, const float* partials, void* ns_ws,
                           bool tensor_cores, const float* W1, const float* W2, const float* W3,
                           float* W1o, float* W2o, float* W3o, __nv_bfloat16_raw* shadow,
                           float* scratch, cudaStream_t st) {
  if (p.ns_steps <= 0 || p.n == 0)
    return reduce_renorm(p, S, partials, W1, W2, W3, W1o, W2o, W3o, shadow, scratch, st);
  const NsWs w = ns_carve(p, ns_ws);
  const int Rp = ns_rows(p.d);
  const int M = 3 * p.H;
  const int tiles = (p.d / 32) * (p.hid / 32);
  {
    TraceScope ts("ns_prepare", st);
    ns_gather_kernel<<<M * tiles, 256, 0, st>>>(partials, S, p.H, p.d, p.hid, Rp, w.X[0],
                                                w.tile_ss);
    ns_scale_kernel<<<dim3(Rp / 8, M), 256, 0, st>>>(p.d, p.hid, Rp, tiles, w.tile_ss, w.X[0],
                                                     w.Xh[0], w.Xl[0]);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (tensor_cores) {
    int* err = device_error_ptr();
    if (err == nullptr) return cudaErrorInvalidDevice;
    e = p.d == 256 ? launch_ns_tc<256, 512>(p, w, err, st) : launch_ns_tc<128, 128>(p, w, err, st);
    if (e != cudaSuccess) return e;
  } else {
    TraceScope ts("ns_f32_iterate", st);
    const size_t xs = (size_t)Rp * p.hid, as = (size_t)Rp * Rp;
    for (int it = 0; it < p.ns_steps; ++it) {
      const float* Xc = w.X[it & 1];
      float* Xn = w.X[(it & 1) ^ 1];
      ns_f32_gemm_kernel<true><<<dim3(Rp / 64, Rp / 64, M), 256, 0, st>>>(
          Xc, Xc, nullptr, w.A, p.hid, p.hid, p.hid, Rp, xs, xs, as, 1.f, 0.f);
      ns_f32_gemm_kernel<false><<<dim3(Rp / 64, Rp / 64, M), 256, 0, st>>>(
          w.A, w.A, w.A, w.B, Rp, Rp, Rp, Rp, as, as, as, kNsC, kNsB);
      ns_f32_gemm_kernel<false><<<dim3(p.hid / 64, Rp / 64, M), 256, 0, st>>>(
          w.B, Xc, Xc, Xn, Rp, Rp, p.hid, p.hid, as, xs, xs, 1.f, kNsA);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  {
    TraceScope ts("ns_finish", st);
    const float* Xf = w.X[p.ns_steps & 1];
    ns_finish_kernel<<<M * tiles, 256, 0, st>>>(Xf, p.H, p.d, p.hid, Rp, w.delta);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return reduce_renorm(p, 1, w.delta, W1, W2, W3, W1o, W2o, W3o, shadow, scratch, st);
}

}  // namespace ttt
