// Work shared by both precisions: the fixed-order reduction of the split-K
// gradient partials, the update W' = W - g and the L2 renormalisation
// (kimjy99 ZipMap review, section 2, the update equations after Eq. 3:
// Ŵ = ‖W‖ (W - Δ)/‖W - Δ‖), plus the bf16 shadow packing.
//
// Renormalisation axis: row-wise by default (each row of W1, W3 of length d,
// each row of W2 of length hidden, to its pre-update norm, no epsilon; a zero
// updated row stays zero); Frobenius (whole matrix per head) or off on request.
// This is HBM-bound CUDA-core work: one warp per row, a sum over the S
// partials in increasing s, and a butterfly sum of squares, so the result is
// the same bit pattern on every run.

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace ttt {

namespace {

__device__ int g_device_error = 0;


__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ __nv_bfloat16_raw to_bf16_raw(float x) {
  __nv_bfloat16 b = __float2bfloat16_rn(x);
  return *reinterpret_cast<__nv_bfloat16_raw*>(&b);
}

// Row decoding: per head, rows [0,hid) are W1, [hid,2hid) W3, [2hid,2hid+d) W2.
struct RowRef {
  int head, blk, row, len;  // blk: 0 = W1, 1 = W3, 2 = W2
};
__device__ __forceinline__ RowRef decode_row(int R, int d, int hid) {
  const int per = 2 * hid + d;
  RowRef r;
  r.head = R / per;
  int x = R % per;
  if (x < hid) {
    r.blk = 0; r.row = x; r.len = d;
  } else if (x < 2 * hid) {
    r.blk = 1; r.row = x - hid; r.len = d;
  } else {
    r.blk = 2; r.row = x - 2 * hid; r.len = hid;
  }
  return r;
}

// V consecutive floats (V = 2 or 4) as one vector access.
template <int V>
__device__ __forceinline__ void load_vec(const float* p, float (&x)[V]) {
  if constexpr (V == 4) {
    const float4 t = *reinterpret_cast<const float4*>(p);
    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
  } else {
    const float2 t = *reinterpret_cast<const float2*>(p);
    x[0] = t.x; x[1] = t.y;
  }
}

// One row of one matrix, handled by one warp.  Lane l holds elements
// 32*V*c + V*l .. +V-1 of the row, c < NC (row length 32*V*NC).  The split
// sum, W' = W -/+ g and both norms are formed in fp64 so that the only
// rounding left on Ŵ - W is the final fp32 store.  Each element sums the S
// partials in increasing s; the row of W and a group of splits (four, or two
// for the longest rows, to bound registers) are loaded before they are summed,
// so a row costs about one memory round trip per group.
template <int V, int NC>
__device__ __forceinline__ void renorm_row(const float* __restrict__ P0, size_t sstride, int S,
                                           const float* W, float* Wo, size_t base, double sign,
                                           int mode, int warp, int lane, __nv_bfloat16_raw* shadow,
                                           double* scratch) {
  float wf[NC][V];
#pragma unroll
  for (int c = 0; c < NC; ++c) load_vec<V>(W + base + 32 * V * c + V * lane, wf[c]);
  double wn[NC][V];
#pragma unroll
  for (int c = 0; c < NC; ++c)
#pragma unroll
    for (int e = 0; e < V; ++e) wn[c][e] = 0.0;
  constexpr int G = NC >= 4 ? 2 : 4;
  for (int s = 0; s < S; s += G) {
    const int g = S - s < G ? S - s : G;
    float x[G][NC][V];
#pragma unroll
    for (int u = 0; u < G; ++u)
      if (u < g)
#pragma unroll
        for (int c = 0; c < NC; ++c) load_vec<V>(P0 + (size_t)(s + u) * sstride + 32 * V * c, x[u][c]);
#pragma unroll
    for (int u = 0; u < G; ++u)
      if (u < g)
#pragma unroll
        for (int c = 0; c < NC; ++c)
#pragma unroll
          for (int e = 0; e < V; ++e) wn[c][e] += (double)x[u][c][e];
  }
  double s_old = 0.0, s_new = 0.0;
#pragma unroll
  for (int c = 0; c < NC; ++c)
#pragma unroll
    for (int e = 0; e < V; ++e) {
      const double w = (double)wf[c][e];
      const double wp = w + sign * wn[c][e];
      wn[c][e] = wp;
      s_old = fma(w, w, s_old);
      s_new = fma(wp, wp, s_new);
    }
  s_old = warp_sum(s_old);
  s_new = warp_sum(s_new);
  double scale = 1.0;
  if (mode == 1) scale = s_new > 0.0 ? sqrt(s_old) / sqrt(s_new) : 1.0;
  if (mode == 2 && lane == 0) {
    scratch[2 * (size_t)warp] = s_old;
    scratch[2 * (size_t)warp + 1] = s_new;
  }
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const size_t idx = base + 32 * V * c + V * lane;
    float v[V];
#pragma unroll
    for (int e = 0; e < V; ++e) v[e] = (float)(wn[c][e] * scale);
    uint32_t pk[V / 2];
#pragma unroll
    for (int e = 0; e < V; e += 2)
      pk[e / 2] = (uint32_t)to_bf16_raw(v[e]).x | ((uint32_t)to_bf16_raw(v[e + 1]).x << 16);
    if constexpr (V == 4) {
      *reinterpret_cast<float4*>(Wo + idx) = make_float4(v[0], v[1], v[2], v[3]);
      if (shadow != nullptr) *reinterpret_cast<uint2*>(shadow + idx) = make_uint2(pk[0], pk[1]);
    } else {
      *reinterpret_cast<float2*>(Wo + idx) = make_float2(v[0], v[1]);
      if (shadow != nullptr) *reinterpret_cast<uint32_t*>(shadow + idx) = pk[0];
    }
  }
}

// nblk = 3: the SwiGLU layer (blocks W1, W3, W2 per head, partials P1 = G1,
// P3 = G3, P2 = -G2).  nblk = 1: linear fast weights (W1 = W, d x d, partial
// P = -g = Σ η v k^T, added).
__global__ void __launch_bounds__(256, 2) reduce_renorm_kernel(
    const float* __restrict__ partials, int S, int H, int d, int hid, int nblk, int mode,
    const float* W1, const float* W2, const float* W3, float* W1o, float* W2o, float* W3o,
    __nv_bfloat16_raw* __restrict__ shadow, double* __restrict__ scratch) {
  grid_dep_launch();
  grid_dep_wait();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int per = nblk == 3 ? 2 * hid + d : d;
  if (warp >= H * per) return;
  RowRef r;
  if (nblk == 3) {
    r = decode_row(warp, d, hid);
  } else {
    r.head = warp / d; r.blk = 0; r.row = warp % d; r.len = d;
  }
  const size_t mat = (size_t)hid * d;
  const float* W = r.blk == 0 ? W1 : r.blk == 1 ? W3 : W2;
  float* Wo = r.blk == 0 ? W1o : r.blk == 1 ? W3o : W2o;
  const size_t base = (size_t)r.head * mat + (size_t)r.row * r.len;
  // P1, P3 are G1, G3 (subtract); P2 is -G2 and the linear P is -g (add).
  const double sign = r.blk == 2 || nblk == 1 ? 1.0 : -1.0;
  const size_t sstride = (size_t)H * nblk * mat;  // one split
  const float* P = partials + ((size_t)r.head * nblk + r.blk) * mat + (size_t)r.row * r.len;
  // the shadow (W1 | W3 | W2 blocks) is written here unless the Frobenius
  // scale still has to be applied
  __nv_bfloat16_raw* sh = shadow != nullptr && mode != 2 ? shadow + (size_t)r.blk * H * mat
                                                         : nullptr;
  // row lengths: d or hidden of a supported shape (64, 128, 256, 512)
  switch (r.len) {
    case 64:
      renorm_row<2, 1>(P + 2 * lane, sstride, S, W, Wo, base, sign, mode, warp, lane, sh, scratch);
      break;
    case 128:
      renorm_row<4, 1>(P + 4 * lane, sstride, S, W, Wo, base, sign, mode, warp, lane, sh, scratch);
      break;
    case 256:
      renorm_row<4, 2>(P + 4 * lane, sstride, S, W, Wo, base, sign, mode, warp, lane, sh, scratch);
      break;
    default:
      renorm_row<4, 4>(P + 4 * lane, sstride, S, W, Wo, base, sign, mode, warp, lane, sh, scratch);
      break;
  }
}

// Frobenius mode: one block per (head, matrix).  Sums the per-row squares in
// row order, then rescales the matrix in place and writes the shadow.
__global__ void __launch_bounds__(256) frob_scale_kernel(
    int H, int d, int hid, int nblk, const double* __restrict__ scratch, float* W1o, float* W2o,
    float* W3o, __nv_bfloat16_raw* __restrict__ shadow) {
  const int head = blockIdx.x / nblk, blk = blockIdx.x % nblk;
  const int per = nblk == 3 ? 2 * hid + d : d;
  const int r0 = head * per + (blk == 0 ? 0 : blk == 1 ? hid : 2 * hid);
  const int rows = blk == 2 ? d : hid;
  __shared__ double sc;
  if (threadIdx.x == 0) {
    double so = 0.0, sn = 0.0;  // sequential, fixed order
    for (int i = 0; i < rows; ++i) {
      so += scratch[2 * (size_t)(r0 + i)];
      sn += scratch[2 * (size_t)(r0 + i) + 1];
    }
    sc = sn > 0.0 ? sqrt(so) / sqrt(sn) : 1.0;
  }
  __syncthreads();
  const size_t mat = (size_t)hid * d;
  float* Wo = (blk == 0 ? W1o : blk == 1 ? W3o : W2o) + (size_t)head * mat;
  __nv_bfloat16_raw* sh = shadow ? shadow + (size_t)blk * H * mat + (size_t)head * mat : nullptr;
  const double s = sc;
  for (size_t i = threadIdx.x; i < mat; i += blockDim.x) {
    const float v = (float)((double)Wo[i] * s);
    Wo[i] = v;
    if (sh) sh[i] = to_bf16_raw(v);
  }
}

__global__ void pack_shadow_kernel(size_t mat_total, const float* __restrict__ W1,
                                   const float* __restrict__ W2, const float* __restrict__ W3,
                                   __nv_bfloat16_raw* __restrict__ shadow) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < mat_total;
       i += (size_t)gridDim.x * blockDim.x) {
    shadow[i] = to_bf16_raw(W1[i]);
    if (W3 != nullptr) shadow[mat_total + i] = to_bf16_raw(W3[i]);
    if (W2 != nullptr) shadow[2 * mat_total + i] = to_bf16_raw(W2[i]);
  }
}

// Fixed-order sum of S split partials (fp64 accumulation), four elements per
// thread so a thread's loads of one split are issued together.
__global__ void __launch_bounds__(256) sum_splits_kernel(const float* __restrict__ partials, int S,
                                                         size_t count, float* __restrict__ out) {
  const size_t q = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) * 4;
  if (q >= count) return;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int s = 0; s < S; ++s) {
    const float4 v = *reinterpret_cast<const float4*>(partials + (size_t)s * count + q);
    acc[0] += v.x;
    acc[1] += v.y;
    acc[2] += v.z;
    acc[3] += v.w;
  }
  *reinterpret_cast<float4*>(out + q) =
      make_float4((float)acc[0], (float)acc[1], (float)acc[2], (float)acc[3]);
}

// Failure-detection self-test: thread 0 waits on an mbarrier nothing will
// complete, through the same bounded wait the kernels use, with a short
// limit; the wait gives up, records kErrSelfTest and the kernel returns.
__global__ void selftest_timeout_kernel(long long limit, int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, err, kErrSelfTest, limit);
}

}  // namespace

cudaError_t reduce_renorm(const Problem& p, int S, const float* partials, const float* W1,
                          const float* W2, const float* W3, float* W1o, float* W2o, float* W3o,
                          __nv_bfloat16_raw* shadow, float* scratch, cudaStream_t st) {
  const int nblk = p.mlp == kMlpLinear ? 1 : 3;
  const int rows = p.H * (nblk == 3 ? 2 * p.hid + p.d : p.d);
  const int blocks = (rows * 32 + 255) / 256;
  TraceScope ts("reduce_renorm", st);
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, reduce_renorm_kernel, partials, S, p.H, p.d,
                                             p.hid, nblk, (int)p.renorm, W1, W2, W3, W1o, W2o,
                                             W3o, shadow, reinterpret_cast<double*>(scratch));
    if (e != cudaSuccess) return e;
  }
  if (p.renorm == 2)
    frob_scale_kernel<<<p.H * nblk, 256, 0, st>>>(p.H, p.d, p.hid, nblk,
                                                 reinterpret_cast<double*>(scratch), W1o, W2o,
                                                 W3o, shadow);
  return cudaGetLastError();
}

cudaError_t sum_splits(int S, size_t count, const float* partials, float* out, cudaStream_t st) {
  // count = 3 * H * hidden * d is a multiple of 4 for every supported shape
  const size_t threads = (count + 3) / 4;
  TraceScope ts("sum_splits", st);
  sum_splits_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(partials, S, count, out);
  return cudaGetLastError();
}

cudaError_t selftest_wait_timeout(long long limit_cycles, cudaStream_t st) {
  int* err = device_error_ptr();
  if (err == nullptr) return cudaErrorInvalidDevice;
  selftest_timeout_kernel<<<1, 32, 0, st>>>(limit_cycles, err);
  return cudaGetLastError();
}

int* device_error_ptr() {
  // Looked up once per device.
  static std::mutex mu;
  static int* addr[64] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<int*>(p);
  }
  return addr[dev];
}

cudaError_t read_and_clear_device_error(int* value) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int));
  if (e != cudaSuccess) return e;
  *value = v;
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
  }
  return e;
}

cudaError_t pack_shadow(int H, int d, int hid, const float* W1, const float* W2,
                        const float* W3, __nv_bfloat16_raw* shadow, cudaStream_t st) {
  const size_t total = (size_t)H * hid * d;
  int blocks = (int)((total + 255) / 256);
  if (blocks > 148 * 8) blocks = 148 * 8;
  TraceScope ts("pack_shadow", st);
  pack_shadow_kernel<<<blocks, 256, 0, st>>>(total, W1, W2, W3, shadow);
  return cudaGetLastError();
}

}  // namespace ttt
