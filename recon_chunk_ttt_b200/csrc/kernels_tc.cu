// bf16 tensor-core path of the TTT update and apply on sm_100a: tcgen05 MMAs
// with fp32 accumulators in tensor memory (TMEM), operands staged in shared
// memory by TMA (cp.async.bulk.tensor, 128-byte swizzle, each CTA loads its own tiles), warp
// specialised (TMA producer, MMA issuer, epilogue warps), every wait bounded.
//
// Update (kimjy99 ZipMap review, section 2, Eq. 1-3): the fused forward /
// backward / token-reduction kernel (kernels_fused.cu, which rounds the fp32
// weights to bf16 on chip) writing one fp32 partial per token split, then the
// shared fixed-order reduce + renorm kernel.
// Apply:        per 128-query tile, for each 64-wide hidden slice:
//               F = Q [W1s; W3s]^T (TMEM), u = SiLU(h1) ⊙ h3 -> bf16 in shared
//               memory, O += u W2s^T (TMEM); hidden activations never leave
//               the SM.

#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc_util.cuh"

namespace ttt {

// Bytes of the update's own workspace (the optional Newton-Schulz region
// follows it).
size_t tc_main_bytes(const Problem& p);

namespace {

constexpr int HS = 64;           // hidden slice per apply step

// A-operand-in-TMEM forms used by the apply: a 128-row x 16-element bf16
// slice of a K-major 128-byte-swizzled shared-memory tile copied into 8 TMEM
// columns (lane = row), and an MMA that reads its A operand from TMEM.
__device__ __forceinline__ void tmem_cp_128x256b(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.128x256b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void umma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// ----------------------------------------------------------------------------
// apply kernel: O = W2 [SiLU(W1 q) ⊙ W3 q], one (query tile, head) per CTA,
// or per cluster of P CTAs when the items are few
// ----------------------------------------------------------------------------
template <int D>
struct AP {
  static constexpr int NCH = D / CH;
  static constexpr int NSTAGE = 4;
  static constexpr int STAGE = 32768;                    // 2 W13 chunks, or one W2 slice
  static constexpr int W13_CH = 2 * HS * CH * 2;         // 16 KB
  static constexpr int CH_PER_STAGE = NCH >= 2 ? 2 : 1;
  static constexpr int OFF_Q = 0;                        // NCH x [128 x 128 B]
  static constexpr int OFF_STAGE = OFF_Q + NCH * BM * 128;
  static constexpr int OFF_U = OFF_STAGE + NSTAGE * STAGE;  // 2 x [128 x 128 B]
  static constexpr int OFF_BAR = OFF_U + 2 * BM * 128;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr int EPI_WARPS = 8;                    // 2 per TMEM lane quadrant
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr uint32_t TMEM_COLS = 512;             // F at 0, q at 128, O at 256
  static constexpr uint32_t TM_Q = 128;                  // the q tile (A of F) in TMEM
};

// Persistent: CTA b takes (query tile, head) items b, b + grid, ...  With
// P > 1 (few items: the launch is one cluster of P CTAs per item) the CTA of
// cluster rank r takes the hidden slices [r nsl / P, (r + 1) nsl / P) of item
// blockIdx.x / P and, once its own MMAs are done, writes its partial O
// (fp32) into its own q and operand buffers; after a cluster barrier the CTA
// of rank o sums rows [o 128 / P, (o + 1) 128 / P) of the P partials in rank
// order (distributed shared memory loads, all P of a row in flight at once)
// into O, and a second barrier keeps every CTA alive until its partial has
// been read.  Per
// item and 64-wide hidden slice js: F(js) = Q [W1s; W3s]^T into TMEM buffer js&1,
// the epilogue turns it into u = SiLU(h1) ⊙ h3 (bf16, shared memory), and
// O += u W2s^T.  The q chunks are released one by one during the
// last slice so the next item's q streams in early; O is drained while the
// next item's first F MMAs run.  The issue order is F(0), F(1), F(2), O(0),
// F(3), O(1), ... so u(js) has two F MMAs' time to be produced.
template <int D>
__global__ void __launch_bounds__(AP<D>::THREADS, 1)
    apply_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mW13,
                 const __grid_constant__ CUtensorMap mW2,
                 int64_t m, int H, int hid, int P, __nv_bfloat16* __restrict__ O, int* err) {
  using L = AP<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* empty = full + L::NSTAGE;
  uint64_t* q_full = empty + L::NSTAGE;  // one per d-chunk
  uint64_t* q_empty = q_full + L::NCH;
  uint64_t* f_full = q_empty + L::NCH;
  uint64_t* f_empty = f_full + 2;
  uint64_t* u_full = f_empty + 2;
  uint64_t* u_empty = u_full + 2;
  uint64_t* o_full = u_empty + 2;
  uint64_t* o_empty = o_full + 1;
  uint64_t* done = o_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nsl = hid / HS;
  const int w13_stages = L::NCH / L::CH_PER_STAGE;
  const int64_t nqt = (m + BM - 1) / BM;
  const int64_t items = nqt * H;
  // this CTA's items (first, first + stride, ...) and hidden slices [js0, js0 + ns)
  const int part = (int)(blockIdx.x % (unsigned)P);
  const int64_t first = blockIdx.x / P, stride = gridDim.x / P;
  const int js0 = part * nsl / P;
  const int ns = (part + 1) * nsl / P - js0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::NSTAGE; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int c = 0; c < L::NCH; ++c) {
      mbar_init(&q_full[c], 1);
      mbar_init(&q_empty[c], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&f_full[b], 1);
      mbar_init(&f_empty[b], L::EPI_WARPS);
      mbar_init(&u_full[b], L::EPI_WARPS);
      mbar_init(&u_empty[b], 1);
    }
    mbar_init(o_full, 1);
    mbar_init(o_empty, L::EPI_WARPS);
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
  grid_dep_launch();
  grid_dep_wait();

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    tma_prefetch_desc(&mQ);
    int stage = 0;
    uint32_t phase = 0;
    int64_t issued = 0, qloads = 0;
    bool ok = true;
    auto next = [&]() -> uint8_t* {
      if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, err, kErrWaitEmpty)) return nullptr;
      return smem + L::OFF_STAGE + stage * L::STAGE;
    };
    auto advance = [&]() {
      ++issued;
      if (++stage == L::NSTAGE) { stage = 0; phase ^= 1; }
    };
    for (int64_t it = first, i = 0; it < items && ok; it += stride, ++i) {
      const int64_t qt = it / H;
      const int head = (int)(it % H);
      for (int c = 0; c < L::NCH && ok; ++c) {
        if (!mbar_wait(&q_empty[c], (uint32_t)(i & 1) ^ 1, abort_flag, err, kErrWaitEmpty)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&q_full[c], BM * 128);
        TTT_DCHECK(qt * BM < m && head * D + (c + 1) * CH <= H * D, err, kErrCheckTma);
        tma_load_2d(smem + L::OFF_Q + c * BM * 128, &mQ, &q_full[c], head * D + c * CH,
                    (int)(qt * BM));
      }
      ++qloads;
      auto load_w13 = [&](int js) {
        for (int g = 0; g < w13_stages && ok; ++g) {
          uint8_t* st = next();
          if (!st) { ok = false; return; }
          mbar_arrive_expect_tx(&full[stage], L::CH_PER_STAGE * L::W13_CH);
          // one box: CH_PER_STAGE d-chunks x {W1s, W3s} x 64 rows
          TTT_DCHECK(head * hid + (js + 1) * HS <= H * hid &&
                         (g + 1) * L::CH_PER_STAGE <= L::NCH, err, kErrCheckTma);
          tma_load_4d(st, &mW13, &full[stage], 0, head * hid + js * HS, 0, g * L::CH_PER_STAGE);
          advance();
        }
      };
      auto load_w2 = [&](int js) {
        uint8_t* st = next();
        if (!st) { ok = false; return; }
        mbar_arrive_expect_tx(&full[stage], D * 128);
        TTT_DCHECK((js + 1) * HS <= hid && head < H, err, kErrCheckTma);
        tma_load_2d(st, &mW2, &full[stage], js * HS, head * D);
        advance();
      };
      for (int js = 0; js < ns && ok; ++js) {
        load_w13(js0 + js);
        if (js >= 2 && ok) load_w2(js0 + js - 2);
      }
      for (int j = ns >= 2 ? ns - 2 : 0; j < ns && ok; ++j) load_w2(js0 + j);
    }
    drain_ring(full, L::NSTAGE, issued, err);
    for (int c = 0; c < L::NCH; ++c) drain_ring(&q_full[c], 1, qloads, err);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idF = idesc_bf16_f32(BM, 2 * HS, false, false);
    const uint32_t idO = idesc_bf16_f32(BM, D, false, false);
    const uint32_t sbase = smem_u32(smem);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    auto take = [&]() -> bool {
      if (!mbar_wait(&full[stage], phase, abort_flag, err, kErrWaitFull)) return false;
      tc_fence_after();
      return true;
    };
    auto release = [&]() {
      umma_commit(&empty[stage]);
      if (++stage == L::NSTAGE) { stage = 0; phase ^= 1; }
    };
    // g = global slice counter: buffer g&1, its (g>>1)-th use.
    auto do_o = [&](int64_t g, int j, int64_t item_i) -> bool {
      const int b = (int)(g & 1);
      const uint32_t par = (uint32_t)((g >> 1) & 1);
      if (!mbar_wait(&u_full[b], par, abort_flag, err, kErrWaitOperand)) return false;
      if (j == 0 &&
          !mbar_wait(o_empty, (uint32_t)(item_i & 1) ^ 1, abort_flag, err, kErrWaitAccFree))
        return false;
      tc_fence_after();
      if (!take()) return false;
      const uint32_t st = sbase + L::OFF_STAGE + stage * L::STAGE;
      const uint32_t ub = sbase + L::OFF_U + b * BM * 128;
#pragma unroll
      for (int kk = 0; kk < HS / 16; ++kk)
        umma_bf16(tmem + 256, sdesc_sw128(ub + kk * KSTEP_BYTES, 16, 1024),
                  sdesc_sw128(st + kk * KSTEP_BYTES, 16, 1024), idO, (j | kk) != 0);
      release();
      umma_commit(&u_empty[b]);
      return true;
    };
    for (int64_t it = first, i = 0; it < items && ok; it += stride, ++i) {
      for (int js = 0; js < ns && ok; ++js) {
        const int64_t g = i * ns + js;
        // one F buffer: wait until the epilogue has drained F(g - 1) (which
        // also means every earlier F MMA, and so every read of the q tile in
        // TMEM, has completed)
        if (!mbar_wait(&f_empty[0], (uint32_t)(g & 1) ^ 1, abort_flag, err, kErrWaitAccFree)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (js == 0) {
          // this item's q tile into TMEM (16 copies of [128 rows x 16 d]);
          // each shared-memory q chunk goes back to the producer once copied
          for (int c = 0; c < L::NCH && ok; ++c) {
            if (!mbar_wait(&q_full[c], (uint32_t)(i & 1), abort_flag, err, kErrWaitFull)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t qa = sbase + L::OFF_Q + c * BM * 128;
#pragma unroll
            for (int kk = 0; kk < CH / 16; ++kk)
              tmem_cp_128x256b(tmem + L::TM_Q + c * 32 + kk * 8,
                               sdesc_sw128(qa + kk * KSTEP_BYTES, 16, 1024));
            umma_commit(&q_empty[c]);
          }
          if (!ok) break;
        }
        for (int gs = 0; gs < w13_stages && ok; ++gs) {
          if (!take()) { ok = false; break; }
          const uint32_t st = sbase + L::OFF_STAGE + stage * L::STAGE;
          for (int cc = 0; cc < L::CH_PER_STAGE; ++cc) {
            const int c = gs * L::CH_PER_STAGE + cc;
#pragma unroll
            for (int kk = 0; kk < CH / 16; ++kk)
              umma_bf16_ta(tmem, tmem + L::TM_Q + c * 32 + kk * 8,
                           sdesc_sw128(st + cc * L::W13_CH + kk * KSTEP_BYTES, 16, 1024), idF,
                           (c | kk) != 0);
          }
          release();
        }
        if (!ok) break;
        umma_commit(&f_full[0]);
        // O lags F by two slices, so the epilogue of slice js has the time of
        // two F MMAs to produce u before the tensor pipe needs it.
        if (js >= 2 && !do_o(g - 2, js - 2, i)) { ok = false; break; }
      }
      if (!ok) break;
      bool tail_ok = true;
      for (int j = ns >= 2 ? ns - 2 : 0; j < ns && tail_ok; ++j)
        tail_ok = do_o(i * ns + j, j, i);
      if (!tail_ok) break;
      umma_commit(o_full);
    }
    umma_commit(done);
    volatile int never = 0;
    mbar_wait(done, 0, &never, err, kErrWaitFinal);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int ch = (warp - 2) / 4;  // hidden columns [32ch, 32ch+32) of a slice
    const int row = q * 32 + lane;
    bool ok = true;
    for (int64_t it = first, i = 0; it < items && ok; it += stride, ++i) {
      const int64_t qt = it / H;
      const int head = (int)(it % H);
      const int64_t qi = qt * BM + row;
      for (int js = 0; js < ns && ok; ++js) {
        const int64_t g = i * ns + js;
        const int b = (int)(g & 1);
        const uint32_t par = (uint32_t)((g >> 1) & 1);
        const bool got = mbar_wait(&f_full[0], (uint32_t)(g & 1), abort_flag, err, kErrWaitAcc);
        __syncwarp();
        if (!got) { ok = false; break; }
        tc_fence_after();
        const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16) + ch * 32;  // the one F buffer
        uint32_t r1[32], r3[32];
        tmem_ld_32x32(tl, r1);
        tmem_ld_32x32(tl + HS, r3);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&f_empty[0]);
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 32; k += 2) {
          const float h1a = __uint_as_float(r1[k]), h1b = __uint_as_float(r1[k + 1]);
          const float ua = h1a * sigmoid_fast(h1a) * __uint_as_float(r3[k]);
          const float ub = h1b * sigmoid_fast(h1b) * __uint_as_float(r3[k + 1]);
          pk[k / 2] = pack_bf16x2(ua, ub);
        }
        if (!mbar_wait(&u_empty[b], par ^ 1, abort_flag, err, kErrWaitOperand)) {
          ok = false;
          break;
        }
        // K-major 128-byte-swizzled row: 16-byte chunk c of row r sits at
        // chunk position c ^ (r % 8).
        uint8_t* urow = smem + L::OFF_U + b * BM * 128 + (row / 8) * 1024 + (row % 8) * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(urow + (((ch * 4 + c) ^ (row % 8)) * 16)) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&u_full[b]);
      }
      if (!ok) break;
      const bool got_o = mbar_wait(o_full, (uint32_t)(i & 1), abort_flag, err, kErrWaitAcc);
      __syncwarp();
      if (!got_o) break;
      if (P > 1) break;  // one item; its partial O leaves after the loop
      tc_fence_after();
      const uint32_t to = tmem + ((uint32_t)(q * 32) << 16) + 256;
      for (int c0 = ch * (D / 2); c0 < (ch + 1) * (D / 2); c0 += 32) {
        uint32_t rr[32];
        tmem_ld_32x32(to + c0, rr);
        tmem_ld_wait();
        if (qi < m) {
          TTT_DCHECK(c0 + 32 <= D && head < H, err, kErrCheckIndex);
          uint4* dst = reinterpret_cast<uint4*>(O + qi * (int64_t)H * D + (int64_t)head * D + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(
                pack_bf16x2(__uint_as_float(rr[8 * v]), __uint_as_float(rr[8 * v + 1])),
                pack_bf16x2(__uint_as_float(rr[8 * v + 2]), __uint_as_float(rr[8 * v + 3])),
                pack_bf16x2(__uint_as_float(rr[8 * v + 4]), __uint_as_float(rr[8 * v + 5])),
                pack_bf16x2(__uint_as_float(rr[8 * v + 6]), __uint_as_float(rr[8 * v + 7])));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_empty);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (P > 1) {
    // This CTA is past its last MMA (its epilogue saw o_full) and its last
    // load (the producer drained its rings): its q and operand buffers are
    // idle.  The partial O goes there, row r at r * D * 4 bytes, fp32,
    // 16-byte chunk c of the row at (c & ~7) | ((c ^ r) & 7).
    tc_fence_after();
    if (warp >= 2) {
      const int q = warp & 3, ch = (warp - 2) / 4, row = q * 32 + lane;
      uint8_t* prow = smem + L::OFF_Q + (size_t)row * D * 4;
      const uint32_t to = tmem + ((uint32_t)(q * 32) << 16) + 256;
      for (int c0 = ch * (D / 2); c0 < (ch + 1) * (D / 2); c0 += 32) {
        uint32_t rr[32];
        tmem_ld_32x32(to + c0, rr);
        tmem_ld_wait();
#pragma unroll
        for (int v = 0; v < 8; ++v)
          *reinterpret_cast<uint4*>(prow + ((c0 / 4) + (v ^ (row & 7))) * 16) =
              make_uint4(rr[4 * v], rr[4 * v + 1], rr[4 * v + 2], rr[4 * v + 3]);
      }
    }
    tc_fence_before();
    // every partial of the cluster is written
    cluster_sync_all();
    const int64_t qt = first / H;
    const int head = (int)(first % H);
    const int r0 = part * BM / P, nr = (part + 1) * BM / P - r0;
    constexpr int VPL = D / 32;  // floats of a row per lane (8 or 2)
    const int nw = (int)(blockDim.x / 32);
    const uint32_t local = smem_u32(smem + L::OFF_Q);
    for (int lr = warp; lr < nr; lr += nw) {
      const int r = r0 + lr;
      const int64_t qi = qt * BM + r;
      if (qi >= m) break;
      // all P loads of the row in flight before the sum
      float x[8][VPL];
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        if (p < P) {
          const uint32_t base = mapa_shared(local, (uint32_t)p) + (uint32_t)r * D * 4;
          if constexpr (VPL == 8) {
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              const int c = 2 * lane + k;
              ld_shared_cluster_v4(base + (uint32_t)(((c & ~7) | ((c ^ r) & 7)) * 16),
                                   &x[p][4 * k]);
            }
          } else {
            const int c = lane >> 1;
            ld_shared_cluster_v2(
                base + (uint32_t)(((c & ~7) | ((c ^ r) & 7)) * 16 + (lane & 1) * 8), x[p]);
          }
        }
      }
      // rank order
      float acc[VPL];
#pragma unroll
      for (int e = 0; e < VPL; ++e) acc[e] = x[0][e];
#pragma unroll
      for (int p = 1; p < 8; ++p)
        if (p < P)
#pragma unroll
          for (int e = 0; e < VPL; ++e) acc[e] += x[p][e];
      TTT_DCHECK(head < H && lane * VPL + VPL <= D, err, kErrCheckIndex);
      __nv_bfloat16* dst = O + qi * (int64_t)H * D + (int64_t)head * D + lane * VPL;
      if constexpr (VPL == 8) {
        *reinterpret_cast<uint4*>(dst) =
            make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                       pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
      } else {
        *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0], acc[1]);
      }
    }
    // no CTA leaves while another may still read its shared memory
    cluster_sync_all();
  }
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

// ----------------------------------------------------------------------------
// Host side
// ----------------------------------------------------------------------------
struct TcWs {
  float *partials, *scratch;
};

// Workspace: the split partials [S][H][3][hid*d] fp32, then the renorm
// scratch.
TcWs carve(const Problem& p, void* ws, int S) {
  TcWs w;
  char* c = static_cast<char*>(ws);
  w.partials = reinterpret_cast<float*>(c);
  c += align_up((size_t)S * p.H * 3 * p.hid * p.d * 4, 1024);
  w.scratch = reinterpret_cast<float*>(c);
  return w;
}

template <int D>
cudaError_t tc_update_impl(const Problem& p, const float* W1, const float* W2, const float* W3,
                           const void* K, const void* V, const float* eta, float* W1o, float* W2o,
                           float* W3o, __nv_bfloat16_raw* shadow, void* ws, cudaStream_t st,
                           float* partial_out) {
  const SplitPlan sp = tc_split_plan(p);
  TcWs w = carve(p, ws, sp.S);
  int* err = device_error_ptr();
  if (err == nullptr) return cudaErrorInvalidDevice;
  if (p.n > 0) {
    const FusedPlan f = fused_plan(p);
    const cudaError_t e =
        fused_update(p, W1, W2, W3, K, V, eta, f, w.partials, err, st);
    if (e != cudaSuccess) return e;
  } else {
    const cudaError_t e =
        cudaMemsetAsync(w.partials, 0, (size_t)sp.S * p.H * 3 * p.hid * p.d * 4, st);
    if (e != cudaSuccess) return e;
  }
  if (partial_out != nullptr)
    return sum_splits(sp.S, (size_t)p.H * 3 * p.hid * p.d, w.partials, partial_out, st);
  return ns_then_renorm(p, sp.S, w.partials, static_cast<char*>(ws) + tc_main_bytes(p), true, W1,
                        W2, W3, W1o, W2o, W3o, shadow, w.scratch, st);
}

// Clusters of P apply CTAs that fit on the current GPU at once (queried once
// per device and P).
template <int D>
int apply_clusters_per_wave(int P) {
  static std::mutex mu;
  static int cache[64][9] = {};
  int dev = 0;
  if (P < 1 || P > 8 || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  std::lock_guard<std::mutex> lk(mu);
  int (&c)[9] = cache[dev];
  if (c[P] == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)P);
    cfg.blockDim = dim3(AP<D>::THREADS);
    cfg.dynamicSmemBytes = AP<D>::SMEM;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)P;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, apply_kernel<D>, &cfg) != cudaSuccess || n < 1) {
      (void)cudaGetLastError();
      n = -1;
    }
    c[P] = n;
  }
  return c[P];
}

// Hidden-slice parts per (query tile, head): 1 (persistent CTAs) unless the
// items fill at most half a wave; then 2, if all the clusters fit on the GPU
// at once.  Measured at 1,374 queries x 4 heads (d 256): 16.8 us with one
// part, 15.1 with two, 15.9 with three (the partial sums cross the cluster
// at about 20 GB/s per SM, which eats the gain of shorter slice chains).
template <int D>
int apply_parts(int64_t items, int nsl) {
  if (nsl >= 2 && 2 * items <= num_sms() && items <= apply_clusters_per_wave<D>(2)) return 2;
  return 1;
}

template <int D>
cudaError_t tc_apply_impl(const Problem& p, const __nv_bfloat16_raw* shadow, const void* Q,
                          void* O, cudaStream_t st) {
  if (p.n == 0) return cudaSuccess;
  int* err = device_error_ptr();
  if (err == nullptr) return cudaErrorInvalidDevice;
  const size_t wsz = (size_t)p.H * p.hid * D;
  const __nv_bfloat16_raw* s1 = shadow;
  const __nv_bfloat16_raw* s3 = shadow + wsz;
  const __nv_bfloat16_raw* s2 = shadow + 2 * wsz;
  CUtensorMap mQ, mW13, mW2;
  const uint64_t ld = (uint64_t)p.H * D;
  {
    const uint64_t dims[2] = {ld, (uint64_t)p.n}, str[1] = {ld * 2};
    const uint32_t box[2] = {CH, BM};
    if (!make_map(&mQ, Q, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    // {64 d, hidden rows of all heads, matrix (W1 | W3), d-chunks}: one box holds,
    // per d-chunk, the 64 rows of W1s followed by the 64 rows of W3s.
    const uint64_t dims[4] = {(uint64_t)CH, (uint64_t)p.H * p.hid, 2, (uint64_t)(D / CH)};
    const uint64_t str[3] = {(uint64_t)D * 2, (uint64_t)(s3 - s1) * 2, CH * 2};
    const uint32_t box[4] = {CH, HS, 2, (uint32_t)AP<D>::CH_PER_STAGE};
    if (!make_map(&mW13, s1, 4, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {(uint64_t)p.hid, (uint64_t)p.H * D}, str[1] = {(uint64_t)p.hid * 2};
    const uint32_t box[2] = {CH, (uint32_t)D};
    if (!make_map(&mW2, s2, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  cudaError_t e = ensure_smem_attr(apply_kernel<D>, AP<D>::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t items = (p.n + BM - 1) / BM * p.H;
  const int P = apply_parts<D>(items, p.hid / HS);
  const int sms = num_sms();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P > 1 ? (unsigned)(items * P) : (unsigned)(items < sms ? items : sms));
  cfg.blockDim = dim3(AP<D>::THREADS);
  cfg.dynamicSmemBytes = AP<D>::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)P;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = P > 1 ? 2 : 1;
  TraceScope ts("tc_apply", st);
  return cudaLaunchKernelEx(&cfg, apply_kernel<D>, mQ, mW13, mW2, p.n, p.H, p.hid, P,
                            static_cast<__nv_bfloat16*>(O), err);
}

}  // namespace

SplitPlan tc_split_plan(const Problem& p) {
  // The fused update's partial slots: see fused_plan.
  const FusedPlan f = fused_plan(p);
  return {f.splits, 0};
}

size_t tc_main_bytes(const Problem& p) {
  const SplitPlan sp = tc_split_plan(p);
  size_t b = align_up((size_t)sp.S * p.H * 3 * p.hid * p.d * 4, 1024);
  b += align_up((size_t)p.H * (2 * p.hid + p.d) * 2 * 8, 1024);
  return b;
}

size_t tc_workspace_bytes(const Problem& p) { return tc_main_bytes(p) + ns_workspace_bytes(p); }

cudaError_t tc_update(const Problem& p, const float* W1, const float* W2, const float* W3,
                      const void* K, const void* V, const float* eta, float* W1o, float* W2o,
                      float* W3o, __nv_bfloat16_raw* shadow, void* ws, cudaStream_t st,
                      float* partial_out) {
  if (p.d == 256)
    return tc_update_impl<256>(p, W1, W2, W3, K, V, eta, W1o, W2o, W3o, shadow, ws, st,
                               partial_out);
  return tc_update_impl<64>(p, W1, W2, W3, K, V, eta, W1o, W2o, W3o, shadow, ws, st,
                            partial_out);
}

cudaError_t tc_apply(const Problem& p, const __nv_bfloat16_raw* shadow, const void* Q, void* O,
                     cudaStream_t st) {
  if (p.d == 256) return tc_apply_impl<256>(p, shadow, Q, O, st);
  return tc_apply_impl<64>(p, shadow, Q, O, st);
}


}  // namespace ttt
