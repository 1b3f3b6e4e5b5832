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
//   ns_scale    fixed-order Frobenius norm, X0 = G / ||G||_F, zero padding
//   iterations  tensor cores: one clustered tcgen05 kernel for all steps;
//               check mode: three fp32 CUDA-core GEMMs per step
//   ns_finish   Delta back to the partials layout (S = 1) for reduce_renorm
//
// Tensor-core precision: a bf16 MMA of plain operands loses too much through
// five quintic steps, so every operand x is split as hi = bf16(x),
// lo = bf16(x - hi) and each product is hi*hi + hi*lo + lo*hi with fp32
// accumulation in TMEM; the iterate itself stays fp32.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

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
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int s = 0; s < S; ++s) {
    const float* P = partials + (((size_t)s * H + head) * 3 + blk) * mat;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty + 8 * i;
      const size_t off = blk < 2 ? (size_t)(j0 + r) * d + c0 + tx : (size_t)(c0 + r) * hid + j0 + tx;
      acc[i] += (double)P[off];
    }
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
                                                       float* __restrict__ X) {
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
  float* Xm = X + (size_t)m * Rp * hid;
  for (int i = threadIdx.x; i < rows_per * hid; i += blockDim.x) {
    const int row = blockIdx.x * rows_per + i / hid, col = i % hid;
    float* x = Xm + (size_t)row * hid + col;
    *x = row < d ? (float)((double)*x * inv) : 0.f;
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
// runs every step; between the three GEMMs of a step the cluster meets at a
// hardware cluster barrier (release/acquire), and operands travel through
// global memory (L2-resident, read with .cg loads).  Per CTA (rank r,
// mi = r / RB, ni = r % RB, RB = Rp / 128):
//   A  = X X^T        tile rows mi*128, cols ni*128  (K = hidden, B K-major)
//   B  = b A + c A A  same tile                      (K = Rp, A symmetric)
//   X' = a X + B X    rows mi*128, cols ni*N3        (K = Rp, X as MN-major B)
// Operands are staged per 64-deep k chunk, fp32 -> (hi, lo) bf16, in the
// 128-byte swizzled layouts the MMA descriptors expect; two stages, the fill
// of one overlapping the MMAs of the other.
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
  static constexpr int TMEM = N3 <= 128 ? 128 : 256;
  static constexpr int THREADS = 256;
  static_assert(N3 % 64 == 0 && N3 <= 256, "X' tile width");
  static_assert(SMEM <= 227 * 1024, "shared memory");
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

// 8 fp32 -> 8 bf16 (hi) and 8 bf16 of the remainders (lo), 16 B each.
__device__ __forceinline__ void split_store(uint8_t* hi, uint8_t* lo, uint32_t off, float4 x0,
                                            float4 x1) {
  const float v[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat16 a = __float2bfloat16_rn(v[2 * i]);
    const __nv_bfloat16 b = __float2bfloat16_rn(v[2 * i + 1]);
    h[i] = pack_bf16x2(__bfloat162float(a), __bfloat162float(b));
    l[i] = pack_bf16x2(v[2 * i] - __bfloat162float(a), v[2 * i + 1] - __bfloat162float(b));
  }
  *reinterpret_cast<uint4*>(hi + off) = make_uint4(h[0], h[1], h[2], h[3]);
  *reinterpret_cast<uint4*>(lo + off) = make_uint4(l[0], l[1], l[2], l[3]);
}

// K-major tile: 128 rows (r0..) x 64 k (k0..) of a row-major fp32 matrix.
// Row r holds 128 bytes; its 16-byte unit u sits at unit u ^ (r & 7).  The
// 1024 units (8 floats each) are split 4 per thread; all loads are issued
// before the first conversion so the L2 round trips overlap.
struct KTile {
  float4 v[4][2];
};
__device__ __forceinline__ void load_kmajor(KTile& t, const float* M, int ld, int r0, int k0) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int u = threadIdx.x + 256 * i;
    const int row = u >> 3, cu = u & 7;
    const float4* src = reinterpret_cast<const float4*>(M + (size_t)(r0 + row) * ld + k0 + cu * 8);
    t.v[i][0] = __ldcg(src);
    t.v[i][1] = __ldcg(src + 1);
  }
}
__device__ __forceinline__ void store_kmajor(const KTile& t, uint8_t* hi, uint8_t* lo) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int u = threadIdx.x + 256 * i;
    const int row = u >> 3, cu = u & 7;
    split_store(hi, lo, row * 128 + ((cu ^ (row & 7)) << 4), t.v[i][0], t.v[i][1]);
  }
}

// MN-major tile: 64 k rows (k0..) x N columns (n0..) of a row-major fp32
// matrix.  Column block nb of 64 sits at nb * 8192; inside it k row k holds
// 128 bytes with unit u at u ^ (k & 7).  64 * N / 8 units, N / 32 per thread.
template <int N>
struct MTile {
  float4 v[N / 32][2];
};
template <int N>
__device__ __forceinline__ void load_mnmajor(MTile<N>& t, const float* M, int ld, int k0, int n0) {
  constexpr int UPR = N / 8;  // 16-byte units per k row
#pragma unroll
  for (int i = 0; i < N / 32; ++i) {
    const int u = threadIdx.x + 256 * i;
    const int k = u / UPR, cn = u % UPR;
    const float4* src = reinterpret_cast<const float4*>(M + (size_t)(k0 + k) * ld + n0 + cn * 8);
    t.v[i][0] = __ldcg(src);
    t.v[i][1] = __ldcg(src + 1);
  }
}
template <int N>
__device__ __forceinline__ void store_mnmajor(const MTile<N>& t, uint8_t* hi, uint8_t* lo) {
  constexpr int UPR = N / 8;
#pragma unroll
  for (int i = 0; i < N / 32; ++i) {
    const int u = threadIdx.x + 256 * i;
    const int k = u / UPR, cn = u % UPR;
    const int nb = cn >> 3, cu = cn & 7;
    split_store(hi, lo, nb * 8192 + k * 128 + ((cu ^ (k & 7)) << 4), t.v[i][0], t.v[i][1]);
  }
}

// acc[TMEM cols 0..N) = A-op (rows a_r0 of Am, K-major) x B-op over `nchunks`
// k chunks of 64.  B-op: rows b_off of Bm (K-major, N = 128) or, when B_MN,
// columns b_off.. of Bm (MN-major).  gchunk counts chunks over the kernel
// (stage = gchunk & 1, use = gchunk >> 1).  Returns with the MMAs in flight;
// the epilogue waits for them.
template <int N, bool B_MN, class L>
__device__ __forceinline__ void ns_gemm(uint8_t* smem, uint64_t* bars, uint32_t tmem, int& gchunk,
                                        int nchunks, const float* Am, int lda, int a_r0,
                                        const float* Bm, int ldb, int b_off,
                                        volatile int* abort, int* err) {
  const uint32_t idesc = idesc_bf16_f32(128, N, false, B_MN);
  for (int j = 0; j < nchunks; ++j, ++gchunk) {
    const int s = gchunk & 1;
    uint8_t* st = smem + s * L::STAGE;
    uint8_t* bst = st + 2 * L::A_T;
    // loads first (registers only), then wait for the stage's previous MMAs
    KTile ta;
    load_kmajor(ta, Am, lda, a_r0, j * 64);
    if constexpr (B_MN) {
      MTile<N> tb;
      load_mnmajor<N>(tb, Bm, ldb, j * 64, b_off);
      if (gchunk >= 2) mbar_wait(&bars[s], ((gchunk >> 1) - 1) & 1, abort, err, kErrWaitEmpty);
      store_kmajor(ta, st, st + L::A_T);
      store_mnmajor<N>(tb, bst, bst + L::B_T);
    } else {
      KTile tb;
      load_kmajor(tb, Bm, ldb, b_off, j * 64);
      if (gchunk >= 2) mbar_wait(&bars[s], ((gchunk >> 1) - 1) & 1, abort, err, kErrWaitEmpty);
      store_kmajor(ta, st, st + L::A_T);
      store_kmajor(tb, bst, bst + L::B_T);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
      const uint32_t a = smem_u32(st), b = smem_u32(bst);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ah = sdesc_sw128(a + kk * 32, 16, 1024);
        const uint64_t al = sdesc_sw128(a + L::A_T + kk * 32, 16, 1024);
        const uint64_t bh = B_MN ? sdesc_sw128(b + kk * 2048, 8192, 1024)
                                 : sdesc_sw128(b + kk * 32, 16, 1024);
        const uint64_t bl = B_MN ? sdesc_sw128(b + L::B_T + kk * 2048, 8192, 1024)
                                 : sdesc_sw128(b + L::B_T + kk * 32, 16, 1024);
        umma_bf16(tmem, ah, bh, idesc, (j | kk) != 0);
        umma_bf16(tmem, ah, bl, idesc, 1);
        umma_bf16(tmem, al, bh, idesc, 1);
      }
      umma_commit(&bars[s]);
    }
  }
}

// Epilogue of one 128 x N tile: warp w reads TMEM lanes 32*(w%4).. (its rows)
// and half (w/4) of the columns.  MODE 0: O = acc; 1: O = b R + c acc;
// 2: O = a R + acc.  R has O's pitch and position.  R is read before the
// wait for the MMAs (chunk `last`), so its round trip overlaps them.
template <int N, int MODE>
__device__ __forceinline__ void ns_epilogue(uint64_t* bars, int last, uint32_t tmem, float* O,
                                            const float* R, int ld, int r0, int c0,
                                            volatile int* abort, int* err) {
  constexpr int HALF = N / 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3, half = warp >> 2;
  const size_t base = (size_t)(r0 + 32 * q + lane) * ld + c0 + half * HALF;
  float4 rv[MODE != 0 ? HALF / 4 : 1];
  if constexpr (MODE != 0) {
#pragma unroll
    for (int i = 0; i < HALF / 4; ++i) rv[i] = __ldcg(reinterpret_cast<const float4*>(R + base) + i);
  }
  mbar_wait(&bars[last & 1], (last >> 1) & 1, abort, err, kErrWaitAcc);
  tc_fence_after();
#pragma unroll
  for (int j = 0; j < HALF / 32; ++j) {
    uint32_t v[32];
    tmem_ld_32x32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(half * HALF + 32 * j), v);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
      float4 x = make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                             __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
      if constexpr (MODE == 1) {
        const float4 y = rv[(32 * j + i) / 4];
        x = make_float4(fmaf(kNsC, x.x, kNsB * y.x), fmaf(kNsC, x.y, kNsB * y.y),
                        fmaf(kNsC, x.z, kNsB * y.z), fmaf(kNsC, x.w, kNsB * y.w));
      } else if constexpr (MODE == 2) {
        const float4 y = rv[(32 * j + i) / 4];
        x = make_float4(fmaf(kNsA, y.x, x.x), fmaf(kNsA, y.y, x.y), fmaf(kNsA, y.z, x.z),
                        fmaf(kNsA, y.w, x.w));
      }
      __stcg(reinterpret_cast<float4*>(O + base + 32 * j + i), x);
    }
  }
  tc_fence_before();
}

template <int CL>
__device__ __forceinline__ void ns_sync() {
  if (CL > 1)
    cluster_barrier();
  else
    __syncthreads();
}

template <int RP, int C>
__global__ void __launch_bounds__(256, 1) ns_tc_kernel(float* X0, float* X1, float* Abuf,
                                                       float* Bbuf, int steps, int* err) {
  using L = NSL<RP, C>;
  extern __shared__ uint8_t ns_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ns_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  const int rank = L::CL > 1 ? (int)cluster_rank() : 0;
  const int m = blockIdx.x / L::CL;
  const int mi = rank / L::RB, ni = rank % L::RB;
  float* Xa = X0 + (size_t)m * RP * C;
  float* Xb = X1 + (size_t)m * RP * C;
  float* A = Abuf + (size_t)m * RP * RP;
  float* B = Bbuf + (size_t)m * RP * RP;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 32) {
    tmem_alloc(tslot, L::TMEM);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  int g = 0;
  for (int it = 0; it < steps; ++it) {
    const float* Xc = (it & 1) ? Xb : Xa;
    float* Xn = (it & 1) ? Xa : Xb;
    ns_gemm<128, false, L>(smem, bars, tmem, g, C / 64, Xc, C, mi * 128, Xc, C, ni * 128,
                           abort_flag, err);
    ns_epilogue<128, 0>(bars, g - 1, tmem, A, nullptr, RP, mi * 128, ni * 128, abort_flag, err);
    ns_sync<L::CL>();
    ns_gemm<128, false, L>(smem, bars, tmem, g, RP / 64, A, RP, mi * 128, A, RP, ni * 128,
                           abort_flag, err);
    ns_epilogue<128, 1>(bars, g - 1, tmem, B, A, RP, mi * 128, ni * 128, abort_flag, err);
    ns_sync<L::CL>();
    ns_gemm<L::N3, true, L>(smem, bars, tmem, g, RP / 64, B, RP, mi * 128, Xc, C, ni * L::N3,
                            abort_flag, err);
    ns_epilogue<L::N3, 2>(bars, g - 1, tmem, Xn, Xc, C, mi * 128, ni * L::N3, abort_flag, err);
    ns_sync<L::CL>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x < 32) {
    __syncwarp();
    tmem_dealloc(tmem, L::TMEM);
  }
}

struct NsWs {
  float *X0, *X1, *A, *B, *delta;
  double* tile_ss;
};

NsWs ns_carve(const Problem& p, void* ws) {
  const int Rp = ns_rows(p.d);
  const size_t M = 3 * (size_t)p.H;
  char* c = static_cast<char*>(ws);
  NsWs w;
  w.X0 = reinterpret_cast<float*>(c);
  c += align_up(M * Rp * p.hid * 4, 1024);
  w.X1 = reinterpret_cast<float*>(c);
  c += align_up(M * Rp * p.hid * 4, 1024);
  w.A = reinterpret_cast<float*>(c);
  c += align_up(M * Rp * Rp * 4, 1024);
  w.B = reinterpret_cast<float*>(c);
  c += align_up(M * Rp * Rp * 4, 1024);
  w.delta = reinterpret_cast<float*>(c);
  c += align_up(M * p.hid * p.d * 4, 1024);
  w.tile_ss = reinterpret_cast<double*>(c);
  return w;
}

template <int RP, int C>
cudaError_t launch_ns_tc(const Problem& p, const NsWs& w, int* err, cudaStream_t st) {
  using L = NSL<RP, C>;
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
  return cudaLaunchKernelEx(&cfg, ns_tc_kernel<RP, C>, w.X0, w.X1, w.A, w.B, p.ns_steps, err);
}

}  // namespace

size_t ns_workspace_bytes(const Problem& p) {
  if (p.ns_steps <= 0) return 0;
  const int Rp = ns_rows(p.d);
  const size_t M = 3 * (size_t)p.H;
  const size_t tiles = (size_t)(p.d / 32) * (p.hid / 32);
  return 2 * align_up(M * Rp * p.hid * 4, 1024) + 2 * align_up(M * Rp * Rp * 4, 1024) +
         align_up(M * p.hid * p.d * 4, 1024) + align_up(M * tiles * 8, 1024);
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
    ns_gather_kernel<<<M * tiles, 256, 0, st>>>(partials, S, p.H, p.d, p.hid, Rp, w.X0, w.tile_ss);
    ns_scale_kernel<<<dim3(Rp / 8, M), 256, 0, st>>>(p.d, p.hid, Rp, tiles, w.tile_ss, w.X0);
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
      const float* Xc = (it & 1) ? w.X1 : w.X0;
      float* Xn = (it & 1) ? w.X0 : w.X1;
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
    const float* Xf = (p.ns_steps & 1) ? w.X1 : w.X0;
    ns_finish_kernel<<<M * tiles, 256, 0, st>>>(Xf, p.H, p.d, p.hid, Rp, w.delta);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return reduce_renorm(p, 1, w.delta, W1, W2, W3, W1o, W2o, W3o, shadow, scratch, st);
}

}  // namespace ttt
