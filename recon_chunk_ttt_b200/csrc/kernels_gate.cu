// Gated output unit on the tensor cores (kimjy99 ZipMap review, section 2
// "Feature Backbone", last equation): o = RMSNorm(o') ⊙ SiLU(W_g o') per head.

#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc_util.cuh"

namespace ttt {
namespace {

// ----------------------------------------------------------------------------
// Gated output unit (ZipMap review, section 2, last equation of "Feature
// Backbone"): o = RMSNorm(o') ⊙ SiLU(W_g o') per head, RMSNorm(x) =
// x / sqrt(mean(x²) + eps).  Persistent: CTA b serves head b % H and token
// tiles b / H, b / H + gridDim / H, ...  W_g of its head ([d out][d in] bf16,
// K-major) stays in shared memory; o' tiles stream through a 4-slot ring of
// [128 x 64] chunks; the gate pre-activation W_g o' accumulates in one of two
// TMEM buffers while the epilogue drains the other.  Two epilogue warps per
// TMEM lane quadrant split a row's columns: each copies its half of the o'
// row out of the ring slots the MMA just consumed (a slot is refilled only
// after the MMA and all epilogue warps released it), the halves' sums of
// squares meet in shared memory (summed in a fixed order), and each warp
// writes its 32 rows x 32 columns of o (bf16) into a private 2 KB buffer
// (64-byte swizzle) and stores them with its own TMA box, so the global
// writes are whole 64-byte row segments.  o may overwrite o': o' is read only
// through TMA, before o of that tile is written, and only its own CTA
// touches the tile.
// ----------------------------------------------------------------------------
template <int D>
struct GT {
  static constexpr int NCH = D / CH;
  static constexpr int WG = D * 128;        // one 64-wide K chunk of W_g: D rows x 128 B
  static constexpr int NSLOT = 4;
  static constexpr int SLOT = BM * 128;     // 16 KB: 128 tokens x 64 d
  static constexpr int OFF_WG = 0;
  static constexpr int OFF_A = OFF_WG + NCH * WG;
  static constexpr int OFF_SS = OFF_A + NSLOT * SLOT;  // [2 parity][2 half][BM] floats
  static constexpr int OFF_OST = OFF_SS + 2 * 2 * BM * 4;  // per epilogue warp: 32 x 64 B
  static constexpr int OST = 32 * 64;
  static constexpr int OFF_BAR = OFF_OST + 8 * OST;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr int EPI_WARPS = 8;       // two per TMEM lane quadrant
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr uint32_t TMEM_COLS = 2 * D <= 128 ? 128 : 2 * D;  // two accumulators
};

template <int D>
__global__ void __launch_bounds__(GT<D>::THREADS, 1)
    gate_kernel(const __grid_constant__ CUtensorMap mWg, const __grid_constant__ CUtensorMap mA,
                const __grid_constant__ CUtensorMap mO, int64_t m, int H, float eps,
                int* err) {
  using L = GT<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* empty = full + L::NSLOT;
  uint64_t* acc_full = empty + L::NSLOT;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* wfull = acc_empty + 2;
  uint64_t* done = wfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int head = (int)(blockIdx.x % H);
  const int64_t t0 = blockIdx.x / H, tstride = gridDim.x / H;
  const int64_t ntiles = (m + BM - 1) / BM;

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::NSLOT; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1 + L::EPI_WARPS);  // MMA commit + every epilogue warp
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], L::EPI_WARPS);
    }
    mbar_init(wfull, 1);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    tma_prefetch_desc(&mA);
    mbar_arrive_expect_tx(wfull, L::NCH * L::WG);
    for (int c = 0; c < L::NCH; ++c)
      tma_load_2d(smem + L::OFF_WG + c * L::WG, &mWg, wfull, c * CH, head * D);
    int slot = 0;
    uint32_t phase = 0;
    int64_t issued = 0;
    bool ok = true;
    for (int64_t t = t0; t < ntiles && ok; t += tstride) {
      for (int c = 0; c < L::NCH; ++c) {
        if (!mbar_wait(&empty[slot], phase ^ 1, abort_flag, err, kErrWaitEmpty)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[slot], L::SLOT);
        TTT_DCHECK(t * BM < m && head * D + (c + 1) * CH <= H * D, err, kErrCheckTma);
        tma_load_2d(smem + L::OFF_A + slot * L::SLOT, &mA, &full[slot], head * D + c * CH,
                    (int)(t * BM));
        ++issued;
        if (++slot == L::NSLOT) { slot = 0; phase ^= 1; }
      }
    }
    drain_ring(full, L::NSLOT, issued, err);
    drain_ring(wfull, 1, 1, err);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = idesc_bf16_f32(BM, D, false, false);
    const uint32_t sbase = smem_u32(smem);
    int slot = 0;
    uint32_t phase = 0;
    bool ok = mbar_wait(wfull, 0, abort_flag, err, kErrWaitFull);
    tc_fence_after();
    for (int64_t t = t0, i = 0; t < ntiles && ok; t += tstride, ++i) {
      const int b = (int)(i & 1);
      if (!mbar_wait(&acc_empty[b], (uint32_t)((i >> 1) & 1) ^ 1, abort_flag, err,
                     kErrWaitAccFree))
        break;
      tc_fence_after();
      for (int c = 0; c < L::NCH; ++c) {
        if (!mbar_wait(&full[slot], phase, abort_flag, err, kErrWaitFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a = sbase + L::OFF_A + slot * L::SLOT;
        const uint32_t w = sbase + L::OFF_WG + c * L::WG;
#pragma unroll
        for (int kk = 0; kk < CH / 16; ++kk)
          umma_bf16(tmem + b * D, sdesc_sw128(a + kk * KSTEP_BYTES, 16, 1024),
                    sdesc_sw128(w + kk * KSTEP_BYTES, 16, 1024), idesc, (c | kk) != 0);
        umma_commit(&empty[slot]);
        if (++slot == L::NSLOT) { slot = 0; phase ^= 1; }
      }
      if (!ok) break;
      umma_commit(&acc_full[b]);
    }
    umma_commit(done);
    volatile int never = 0;
    mbar_wait(done, 0, &never, err, kErrWaitFinal);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    constexpr int HALF = D / 2;
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const size_t ld = (size_t)H * D;
    float* ss_part = reinterpret_cast<float*>(smem + L::OFF_SS);
    uint8_t* ost = smem + L::OFF_OST + (warp - 2) * L::OST;
    for (int64_t t = t0, i = 0; t < ntiles; t += tstride, ++i) {
      const int b = (int)(i & 1);
      const int64_t r = t * BM + row;
      const bool valid = r < m;
      const bool got = mbar_wait(&acc_full[b], (uint32_t)((i >> 1) & 1), abort_flag, err,
                                 kErrWaitAcc);
      // this half of the o' row from the tile's ring slots: chunk c of tile i
      // sits in slot (i*NCH + c) % NSLOT, 128-byte rows, 16-byte unit u of
      // row r at unit u ^ (r % 8); the chunk's full barrier (already
      // complete) makes the TMA data visible to this thread
      uint4 ov[HALF / 8];
#pragma unroll
      for (int v = 0; v < HALF / 8; ++v) {
        const int col = half * HALF + 8 * v;
        const int c = col / CH, u = (col % CH) / 8;
        const int64_t cg = i * L::NCH + c;
        const int slot = (int)(cg % L::NSLOT);
        if (got && (v == 0 || (col % CH) == 0))
          mbar_wait(&full[slot], (uint32_t)((cg / L::NSLOT) & 1), abort_flag, err, kErrWaitFull);
        ov[v] = *reinterpret_cast<const uint4*>(smem + L::OFF_A + slot * L::SLOT + row * 128 +
                                                ((u ^ (row & 7)) << 4));
      }
      // release the tile's slots (this warp's share)
      __syncwarp();
      if (lane == 0)
        for (int c = 0; c < L::NCH; ++c) mbar_arrive(&empty[(int)((i * L::NCH + c) % L::NSLOT)]);
      float ss = 0.f;
#pragma unroll
      for (int v = 0; v < HALF / 8; ++v) {
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&ov[v]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h2[e]);
          ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
        }
      }
      ss_part[((b * 2) + half) * BM + row] = ss;
      // the pair meets here: partial sums visible, and a failed wait in either
      // warp sends both out together
      if (named_bar_any(1 + q, 64, !got)) break;
      tc_fence_after();
      const float tot = ss_part[(b * 2 + 0) * BM + row] + ss_part[(b * 2 + 1) * BM + row];
      const float inv = rsqrtf(tot / (float)D + eps);
#pragma unroll
      for (int g = 0; g < HALF / 32; ++g) {
        uint32_t acc[32];
        TTT_DCHECK(b * D + half * HALF + 32 * g + 32 <= (int)L::TMEM_COLS, err, kErrCheckTmem);
        tmem_ld_32x32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * D + half * HALF + 32 * g),
                      acc);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&ov[(32 * g + e) / 8]);
          const float2 o = __bfloat1622float2(h2[(e % 8) / 2]);
          const float g0 = __uint_as_float(acc[e]), g1 = __uint_as_float(acc[e + 1]);
          pk[e / 2] = pack_bf16x2(o.x * inv * g0 * sigmoid_fast(g0),
                                  o.y * inv * g1 * sigmoid_fast(g1));
        }
        // this warp's [32 rows x 32 columns] of o through its staging buffer
        // (64-byte swizzle: 16-byte unit c of row r at c ^ ((r / 2) % 4))
        if (lane == 0) bulk_wait_group_read0();  // the previous box has been read
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(ost + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4)) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        TTT_DCHECK(head * D + half * HALF + 32 * g + 32 <= H * D, err, kErrCheckTma);
        if (lane == 0 && t * BM + 32 * q < m) {  // rows past m are clipped by the store
          tma_store_2d(&mO, ost, head * D + half * HALF + 32 * g, (int)(t * BM) + 32 * q);
          bulk_commit_group();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
    if (lane == 0) bulk_wait_group0();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

template <int D>
cudaError_t tc_gate_impl(const Problem& p, const __nv_bfloat16* Wg, const void* Oin, void* Oout,
                         float eps, cudaStream_t st) {
  if (p.n == 0) return cudaSuccess;
  int* err = device_error_ptr();
  if (err == nullptr) return cudaErrorInvalidDevice;
  CUtensorMap mWg, mA, mO;
  {
    const uint64_t dims[2] = {(uint64_t)D, (uint64_t)p.H * D}, str[1] = {(uint64_t)D * 2};
    const uint32_t box[2] = {CH, (uint32_t)D};
    if (!make_map(&mWg, Wg, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t ld = (uint64_t)p.H * D;
    const uint64_t dims[2] = {ld, (uint64_t)p.n}, str[1] = {ld * 2};
    const uint32_t box[2] = {CH, BM};
    const uint32_t obox[2] = {32, 32};
    if (!make_map(&mA, Oin, 2, dims, str, box) ||
        !make_map(&mO, Oout, 2, dims, str, obox, CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
  }
  cudaError_t e = ensure_smem_attr(gate_kernel<D>, GT<D>::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (p.n + BM - 1) / BM;
  const int per_head = num_sms() / p.H;
  const int64_t ctas_per_head = tiles < per_head ? tiles : (per_head > 0 ? per_head : 1);
  const unsigned grid = (unsigned)(ctas_per_head * p.H);
  {
    TraceScope ts("tc_gate", st);
    gate_kernel<D><<<grid, GT<D>::THREADS, GT<D>::SMEM, st>>>(
        mWg, mA, mO, p.n,
        p.H, eps, err);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t tc_gate(const Problem& p, const void* Wg, const void* Oin, void* Oout, float eps,
                    cudaStream_t st) {
  const auto* w = static_cast<const __nv_bfloat16*>(Wg);
  if (p.d == 256) return tc_gate_impl<256>(p, w, Oin, Oout, eps, st);
  return tc_gate_impl<64>(p, w, Oin, Oout, eps, st);
}

}  // namespace ttt
