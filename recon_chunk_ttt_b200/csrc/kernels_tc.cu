// bf16 tensor-core path of the TTT update and apply on sm_100a: tcgen05 MMAs
// with fp32 accumulators in tensor memory (TMEM), operands staged in shared
// memory by TMA (cp.async.bulk.tensor, 128-byte swizzle, each CTA loads its own tiles), warp
// specialised (one TMA producer thread, one MMA issuer thread, epilogue
// warps), every wait bounded.
//
// Update of one head (kimjy99 ZipMap review, section 2, Eq. 1-3):
//   fb kernel   h1 = W1 k, h3 = W3 k (one N=128 MMA over [W1s; W3s]),
//               du = -W2^T v (N=64 MMA), then in the epilogue
//               η·u, η·dh1, η·dh3 (u = SiLU(h1) ⊙ h3, dh3 = du ⊙ SiLU(h1),
//               dh1 = du ⊙ h3 ⊙ SiLU'(h1)) stored as bf16 [H][n][hid].
//   grad kernel split-K token reduction on MN-major operands:
//               P1 = Σ η dh1 k^T, P3 = Σ η dh3 k^T, P2 = Σ η u v^T (= -G2^T,
//               stored transposed as [d][hid]); fixed token ranges.
//   then the shared fixed-order reduce + renorm kernel.
// Apply:        per 128-query tile, for each 64-wide hidden slice:
//               F = Q [W1s; W3s]^T (TMEM), u = SiLU(h1) ⊙ h3 -> bf16 in shared
//               memory, O += u W2s^T (TMEM); hidden activations never leave
//               the SM.

#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc_util.cuh"

namespace ttt {

// Bytes of the update's own workspace (the optional Newton-Schulz region
// follows it).
size_t tc_main_bytes(const Problem& p);

namespace {

constexpr int HS = 64;           // hidden slice per fb CTA / apply step
constexpr int TK = 64;           // tokens per grad stage

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
// Weight prologue: bf16 copies of W1, W3 ([H][hid][d]) and of W2^T ([H][hid][d])
// ----------------------------------------------------------------------------
__global__ void convert_weights_kernel(int H, int d, int hid, const float* __restrict__ W1,
                                       const float* __restrict__ W2, const float* __restrict__ W3,
                                       __nv_bfloat16* __restrict__ b1, __nv_bfloat16* __restrict__ b3,
                                       __nv_bfloat16* __restrict__ b2t) {
  // One block per 32 x 32 tile (hidden rows j0.., d columns c0..) of one head;
  // the W2 tile is transposed through shared memory so that both its read and
  // its write are coalesced.
  __shared__ float tile[32][33];
  const int tiles_c = d / 32, tiles_j = hid / 32;
  const int h = blockIdx.x / (tiles_c * tiles_j);
  const int t = blockIdx.x % (tiles_c * tiles_j);
  const int j0 = (t / tiles_c) * 32, c0 = (t % tiles_c) * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const size_t mat = (size_t)h * hid * d;
  for (int r = ty; r < 32; r += 8) {
    const size_t i = mat + (size_t)(j0 + r) * d + c0 + tx;
    b1[i] = __float2bfloat16_rn(W1[i]);
    b3[i] = __float2bfloat16_rn(W3[i]);
    tile[r][tx] = W2[mat + (size_t)(c0 + r) * hid + j0 + tx];
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8)
    b2t[mat + (size_t)(j0 + r) * d + c0 + tx] = __float2bfloat16_rn(tile[tx][r]);
}

// ----------------------------------------------------------------------------
// fb kernel: forward dual GEMM + backward GEMM + gated epilogue
// ----------------------------------------------------------------------------
template <int D>
struct FB {
  static constexpr int NCH = D / CH;
  static constexpr int CPS = NCH >= 2 ? 2 : 1;            // d-chunks per stage (one TMA box)
  static constexpr int NSTAGE = 6 / CPS;
  static constexpr int CHUNK = BM * CH * 2;               // 16 KB: 128 tokens x 64 d
  static constexpr int STAGE = CPS * CHUNK;
  static constexpr int W13_CH = 2 * HS * CH * 2;          // 16 KB: W1s rows then W3s rows
  static constexpr int W2_CH = HS * CH * 2;               // 8 KB
  static constexpr int OUT_TILE = BM * HS * 2;            // 16 KB: one output [128 x 64] bf16
  static constexpr int OFF_W13 = 0;
  static constexpr int OFF_W2 = OFF_W13 + NCH * W13_CH;
  static constexpr int OFF_STAGE = OFF_W2 + NCH * W2_CH;
  static constexpr int OFF_OUT = OFF_STAGE + NSTAGE * STAGE;  // 2 rotating output boxes
  static constexpr int OFF_BAR = OFF_OUT + 2 * OUT_TILE;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;       // + alignment slack
  static constexpr int EPI_WARPS = 8;                     // 2 per TMEM lane quadrant
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;     // producer, MMA, epilogue
  static constexpr uint32_t TMEM_COLS = 512;              // 2 x (F13 128 + DU 64), at 0 / 256
};

// Work items are (head*nslices + slice, token tile) pairs.  With reps > 0 the
// grid is groups*reps CTAs: CTA b owns group b / reps and the token tiles
// [r*ntiles/reps, (r+1)*ntiles/reps), r = b % reps, so the hidden slices of one
// head walk the same k/v tiles in lockstep and share them through L2.  With
// reps == 0 (more groups than CTAs) each CTA takes a contiguous range of the
// flattened item space.
__device__ __forceinline__ void fb_item_range(int64_t ntiles, int groups, int reps,
                                              int64_t& it0, int64_t& it1) {
  if (reps > 0) {
    const int64_t g = blockIdx.x / reps, r = blockIdx.x % reps;
    it0 = g * ntiles + r * ntiles / reps;
    it1 = g * ntiles + (r + 1) * ntiles / reps;
  } else {
    const int64_t total = (int64_t)groups * ntiles;
    it0 = total * blockIdx.x / gridDim.x;
    it1 = total * (blockIdx.x + 1) / gridDim.x;
  }
}

template <int D>
__global__ void __launch_bounds__(FB<D>::THREADS, 1)
    fb_kernel(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
              const __grid_constant__ CUtensorMap mW1, const __grid_constant__ CUtensorMap mW3,
              const __grid_constant__ CUtensorMap mW2t, const __grid_constant__ CUtensorMap mUs,
              const __grid_constant__ CUtensorMap mD1s, const __grid_constant__ CUtensorMap mD3s,
              const float* __restrict__ eta, int64_t n, int H, int hid, int reps, int* err) {
  using L = FB<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* empty = full + L::NSTAGE;
  uint64_t* wfull = empty + L::NSTAGE;
  uint64_t* wempty = wfull + 1;
  uint64_t* acc_full = wempty + 1;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nslices = hid / HS;
  const int64_t ntiles = (n + BM - 1) / BM;
  int64_t it0, it1;
  fb_item_range(ntiles, H * nslices, reps, it0, it1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(wfull, 1);
    mbar_init(wempty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], L::EPI_WARPS);
    }
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
    tma_prefetch_desc(&mK);
    tma_prefetch_desc(&mV);
    int stage = 0;
    uint32_t phase = 0, wphase = 0;
    int cur_hs = -1;
    int64_t issued = 0, wloads = 0;
    bool ok = true;
    for (int64_t it = it0; it < it1 && ok; ++it) {
      const int hs = (int)(it / ntiles);
      const int64_t tile = it % ntiles;
      const int head = hs / nslices, slice = hs % nslices;
      if (hs != cur_hs) {
        if (cur_hs >= 0) {
          if (!mbar_wait(wempty, wphase, abort_flag, err, kErrWaitEmpty)) { ok = false; break; }
          wphase ^= 1;
        }
        mbar_arrive_expect_tx(wfull, L::NCH * (L::W13_CH + L::W2_CH));
        const int row = head * hid + slice * HS;
        TTT_DCHECK(row >= 0 && row + HS <= H * hid, err, kErrCheckTma);
        for (int c = 0; c < L::NCH; ++c) {
          uint8_t* w13 = smem + L::OFF_W13 + c * L::W13_CH;
          tma_load_2d(w13, &mW1, wfull, c * CH, row);
          tma_load_2d(w13 + HS * 128, &mW3, wfull, c * CH, row);
          tma_load_2d(smem + L::OFF_W2 + c * L::W2_CH, &mW2t, wfull, c * CH, row);
        }
        ++wloads;
        cur_hs = hs;
      }
      const int y = (int)(tile * BM);
      for (int pass = 0; pass < 2 && ok; ++pass) {
        const CUtensorMap* m = pass == 0 ? &mK : &mV;
        for (int g = 0; g < L::NCH / L::CPS; ++g) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, err, kErrWaitEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], L::STAGE);
          TTT_DCHECK(y >= 0 && (int64_t)y < n && head * L::NCH + (g + 1) * L::CPS <= H * L::NCH,
                     err, kErrCheckTma);
          // one box = CPS chunks of [128 tokens x 64 d]
          tma_load_3d(smem + L::OFF_STAGE + stage * L::STAGE, m, &full[stage], 0, y,
                      head * L::NCH + g * L::CPS);
          ++issued;
          if (++stage == L::NSTAGE) { stage = 0; phase ^= 1; }
        }
      }
    }
    drain_ring(full, L::NSTAGE, issued, err);
    drain_ring(wfull, 1, wloads, err);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idF = idesc_bf16_f32(BM, 2 * HS, false, false);
    const uint32_t idU = idesc_bf16_f32(BM, HS, false, false);
    int stage = 0;
    uint32_t phase = 0, wphase = 0;
    uint32_t abits = 0;  // bit b: phase parity of accumulator buffer b
    int cur_hs = -1, buf = 0;
    bool ok = true;
    const uint32_t sbase = smem_u32(smem);
    for (int64_t it = it0; it < it1 && ok; ++it) {
      const int hs = (int)(it / ntiles);
      if (hs != cur_hs) {
        if (cur_hs >= 0) umma_commit(wempty);  // old weights free once prior MMAs finish
        if (!mbar_wait(wfull, wphase, abort_flag, err, kErrWaitFull)) { ok = false; break; }
        wphase ^= 1;
        cur_hs = hs;
      }
      if (!mbar_wait(&acc_empty[buf], ((abits >> buf) & 1) ^ 1, abort_flag, err,
                     kErrWaitAccFree)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t dF = tmem + buf * 256, dU = tmem + buf * 256 + 128;
      for (int pass = 0; pass < 2 && ok; ++pass) {
        for (int g = 0; g < L::NCH / L::CPS; ++g) {
          if (!mbar_wait(&full[stage], phase, abort_flag, err, kErrWaitFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int cc = 0; cc < L::CPS; ++cc) {
            const int c = g * L::CPS + cc;
            const uint32_t a = sbase + L::OFF_STAGE + stage * L::STAGE + cc * L::CHUNK;
            const uint32_t b = pass == 0 ? sbase + L::OFF_W13 + c * L::W13_CH
                                         : sbase + L::OFF_W2 + c * L::W2_CH;
#pragma unroll
            for (int kk = 0; kk < CH / 16; ++kk) {
              const uint64_t da = sdesc_sw128(a + kk * KSTEP_BYTES, 16, 1024);
              const uint64_t db = sdesc_sw128(b + kk * KSTEP_BYTES, 16, 1024);
              umma_bf16(pass == 0 ? dF : dU, da, db, pass == 0 ? idF : idU, (c | kk) != 0);
            }
          }
          umma_commit(&empty[stage]);
          if (++stage == L::NSTAGE) { stage = 0; phase ^= 1; }
        }
      }
      umma_commit(&acc_full[buf]);
      abits ^= 1u << buf;
      buf ^= 1;
    }
    // Wait for every MMA issued by this thread before TMEM is released.
    umma_commit(done);
    volatile int never = 0;
    mbar_wait(done, 0, &never, err, kErrWaitFinal);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    // Two warps per TMEM lane quadrant; warp half `ch` takes hidden columns
    // [32*ch, 32*ch+32) of the slice.  Outputs are staged in shared memory in
    // the 128-byte-swizzled box layout and written by TMA bulk stores.
    const int q = warp & 3;
    const int ch = (warp - 2) / 4;
    const int row = q * 32 + lane;
    const bool leader = warp == 2 && lane == 0;
    uint8_t* stage_out = smem + L::OFF_OUT;
    uint32_t out_k = 0;  // stores issued so far (selects the staging buffer)
    uint32_t abits = 0;
    int buf = 0;
    for (int64_t it = it0; it < it1; ++it) {
      const int hs = (int)(it / ntiles);
      const int64_t tile = it % ntiles;
      const int head = hs / nslices, slice = hs % nslices;
      const int64_t tok = tile * BM + row;
      const bool live = tok < n;
      const float ne = live ? -__ldg(&eta[tok * H + head]) : 0.f;  // -η: du = -(W2^T v)
      const bool got =
          mbar_wait(&acc_full[buf], (abits >> buf) & 1, abort_flag, err, kErrWaitAcc);
      __syncwarp();
      if (named_bar_any(1, 32 * L::EPI_WARPS, !got)) break;
      abits ^= 1u << buf;
      tc_fence_after();
      const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16) + buf * 256 + ch * 32;
      TTT_DCHECK(buf * 256 + ch * 32 + 128 + 32 <= (int)L::TMEM_COLS, err, kErrCheckTmem);
      uint32_t r1[32], r3[32], rd[32];
      tmem_ld_32x32(tl, r1);
      tmem_ld_32x32(tl + HS, r3);
      tmem_ld_32x32(tl + 128, rd);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      uint32_t pk[3][16];  // η·u, η·dh1, η·dh3 as packed bf16 pairs
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        float o_u[2], o_1[2], o_3[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float h1 = __uint_as_float(r1[i + e]);
          const float h3 = __uint_as_float(r3[i + e]);
          const float edu = ne * __uint_as_float(rd[i + e]);  // η du
          const float s = sigmoid_fast(h1);
          const float a = h1 * s;                             // SiLU(h1)
          const float dsl = fmaf(-a, s, a + s);               // SiLU'(h1) = s + a(1-s)
          o_u[e] = -ne * (a * h3);
          o_3[e] = edu * a;
          o_1[e] = edu * h3 * dsl;
        }
        pk[0][i / 2] = pack_bf16x2(o_u[0], o_u[1]);
        pk[1][i / 2] = pack_bf16x2(o_1[0], o_1[1]);
        pk[2][i / 2] = pack_bf16x2(o_3[0], o_3[1]);
      }
      // Three [128 x 64] boxes go out through two rotating staging buffers;
      // before refilling one, the store issued from it two stores ago must
      // have finished reading it.
      const int x = slice * HS, y = (int)(tile * BM);
      TTT_DCHECK(x + HS <= hid && (int64_t)y < n, err, kErrCheckTma);
#pragma unroll
      for (int o = 0; o < 3; ++o) {
        uint8_t* box = stage_out + (out_k & 1) * L::OUT_TILE;
        if (leader) bulk_wait_group_read1();
        named_bar_sync(1, 32 * L::EPI_WARPS);
        uint8_t* r = box + (row / 8) * 1024 + (row % 8) * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(r + (((ch * 4 + c) ^ (row % 8)) * 16)) =
              make_uint4(pk[o][4 * c], pk[o][4 * c + 1], pk[o][4 * c + 2], pk[o][4 * c + 3]);
        fence_proxy_async_smem();
        named_bar_sync(1, 32 * L::EPI_WARPS);
        if (leader) {
          tma_store_3d(o == 0 ? &mUs : o == 1 ? &mD1s : &mD3s, box, x, y, head);
          bulk_commit_group();
        }
        ++out_k;
      }
      buf ^= 1;
    }
    if (leader) bulk_wait_group0();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

// ----------------------------------------------------------------------------
// grad kernel: split-K token reduction with MN-major operands
//   kind 0: acc0 = Σ_t DH1[t, tile]^T K[t, :], acc1 = Σ_t DH3[t, tile]^T K[t, :]
//   kind 1: acc_a = Σ_t U[t, tile_a]^T V[t, :] for two hidden tiles (one if
//           hid = 128)
// Each CTA = (kind, head, hidden tile group, split s); split s owns tokens
// [s*chunk, min(n, (s+1)*chunk)), chunk a multiple of TK.
// ----------------------------------------------------------------------------
template <int D>
struct GR {
  static constexpr int NSTAGE = 3;
  static constexpr int A_TILE = BM * TK * 2;              // 16 KB: 2 boxes [64 tok x 64 hid]
  static constexpr int B_TILE = D * TK * 2;               // D/64 boxes [64 tok x 64 d]
  static constexpr int STAGE = 2 * A_TILE + B_TILE;
  static constexpr int OFF_BAR = NSTAGE * STAGE;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 512;              // acc a at column a*256
};

template <int D>
__global__ void __launch_bounds__(GR<D>::THREADS, 1)
    grad_kernel(const __grid_constant__ CUtensorMap mDH1, const __grid_constant__ CUtensorMap mDH3,
                const __grid_constant__ CUtensorMap mU, const __grid_constant__ CUtensorMap mK,
                const __grid_constant__ CUtensorMap mV, int64_t n, int H, int hid, int64_t chunk,
                int ctas_kind0, int ctas_kind1, float* __restrict__ partials, int* err) {
  using L = GR<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* empty = full + L::NSTAGE;
  uint64_t* acc_full = empty + L::NSTAGE;
  uint64_t* done = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // Decode (split, kind, head, tile group).
  const int per_split = ctas_kind0 + ctas_kind1;
  const int s = blockIdx.x / per_split;
  int r = blockIdx.x % per_split;
  const int kind = r < ctas_kind0 ? 0 : 1;
  if (kind == 1) r -= ctas_kind0;
  const int groups_per_head = kind == 0 ? hid / BM : (hid / BM + 1) / 2;
  const int head = r / groups_per_head, grp = r % groups_per_head;
  const int j_first = kind == 0 ? grp * BM : grp * 2 * BM;
  const int nacc = kind == 0 ? 2 : (j_first + BM < hid ? 2 : 1);
  const int64_t ts = (int64_t)s * chunk;
  const int64_t te = ts + chunk < n ? ts + chunk : n;
  const int nsteps = te > ts ? (int)((te - ts + TK - 1) / TK) : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::NSTAGE; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
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
    int stage = 0;
    uint32_t phase = 0;
    int64_t issued = 0;
    const uint32_t bytes = (uint32_t)(nacc * L::A_TILE + L::B_TILE);
    for (int k = 0; k < nsteps; ++k) {
      if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, err, kErrWaitEmpty)) break;
      uint8_t* st = smem + stage * L::STAGE;
      mbar_arrive_expect_tx(&full[stage], bytes);
      const int y = (int)(ts + (int64_t)k * TK);
      for (int a = 0; a < nacc; ++a) {
        const CUtensorMap* m = kind == 0 ? (a == 0 ? &mDH1 : &mDH3) : &mU;
        const int j = kind == 0 ? j_first : j_first + a * BM;
        // one box: 2 hidden chunks x [64 tokens x 64 hidden]
        tma_load_4d(st + a * L::A_TILE, m, &full[stage], 0, y, j / CH, head);
      }
      // one box: D/64 d-chunks x [64 tokens x 64 d]
      tma_load_3d(st + 2 * L::A_TILE, kind == 0 ? &mK : &mV, &full[stage], 0, y, head * (D / CH));
      ++issued;
      if (++stage == L::NSTAGE) { stage = 0; phase ^= 1; }
    }
    drain_ring(full, L::NSTAGE, issued, err);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = idesc_bf16_f32(BM, D, true, true);
    const uint32_t sbase = smem_u32(smem);
    int stage = 0;
    uint32_t phase = 0;
    for (int k = 0; k < nsteps; ++k) {
      if (!mbar_wait(&full[stage], phase, abort_flag, err, kErrWaitFull)) break;
      tc_fence_after();
      const uint32_t st = sbase + stage * L::STAGE;
#pragma unroll
      for (int kk = 0; kk < TK / 16; ++kk) {
        // 16 tokens = two 8-row groups of 1024 bytes.
        const uint64_t db = sdesc_sw128(st + 2 * L::A_TILE + kk * 2048, TK * 128, 1024);
        for (int a = 0; a < nacc; ++a) {
          const uint64_t da = sdesc_sw128(st + a * L::A_TILE + kk * 2048, TK * 128, 1024);
          umma_bf16(tmem + a * 256, da, db, idesc, (k | kk) != 0);
        }
      }
      umma_commit(&empty[stage]);
      if (++stage == L::NSTAGE) { stage = 0; phase ^= 1; }
    }
    umma_commit(acc_full);
    umma_commit(done);
    volatile int never = 0;
    mbar_wait(done, 0, &never, err, kErrWaitFinal);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const bool have = nsteps > 0 && mbar_wait(acc_full, 0, abort_flag, err, kErrWaitAcc);
    __syncwarp();
    tc_fence_after();
    const size_t mat = (size_t)hid * D;
    for (int a = 0; a < nacc; ++a) {
      const int blk = kind == 0 ? a : 2;  // P1, P3, P2
      float* P = partials + (((size_t)s * H + head) * 3 + blk) * mat;
      const int j = (kind == 0 ? j_first : j_first + a * BM) + q * 32 + lane;
      TTT_DCHECK(j < hid && a * 256 + D <= (int)L::TMEM_COLS, err, kErrCheckIndex);
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t rr[32];
        if (have) {
          tmem_ld_32x32(tmem + ((uint32_t)(q * 32) << 16) + a * 256 + c0, rr);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) rr[i] = 0u;
        }
        if (kind == 0) {
          float4* dst = reinterpret_cast<float4*>(P + (size_t)j * D + c0);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_float4(__uint_as_float(rr[4 * v]), __uint_as_float(rr[4 * v + 1]),
                                 __uint_as_float(rr[4 * v + 2]), __uint_as_float(rr[4 * v + 3]));
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) P[(size_t)(c0 + i) * hid + j] = __uint_as_float(rr[i]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

// ----------------------------------------------------------------------------
// apply kernel: O = W2 [SiLU(W1 q) ⊙ W3 q], one (query tile, head) per CTA
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

// Persistent: CTA b takes (query tile, head) items b, b + grid, ...  Per item
// and 64-wide hidden slice js: F(js) = Q [W1s; W3s]^T into TMEM buffer js&1,
// the epilogue turns it into u = SiLU(h1) ⊙ h3 (bf16, shared memory), and
// O += u W2s^T.  The q chunks are released one by one during the
// last slice so the next item's q streams in early; O is drained while the
// next item's first F MMAs run.  The issue order is F(0), F(1), F(2), O(0),
// F(3), O(1), ... so u(js) has two F MMAs' time to be produced.
template <int D>
__global__ void __launch_bounds__(AP<D>::THREADS, 1)
    apply_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mW13,
                 const __grid_constant__ CUtensorMap mW2,
                 int64_t m, int H, int hid, __nv_bfloat16* __restrict__ O, int* err) {
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
    for (int64_t it = blockIdx.x, i = 0; it < items && ok; it += gridDim.x, ++i) {
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
      for (int js = 0; js < nsl && ok; ++js) {
        load_w13(js);
        if (js >= 2 && ok) load_w2(js - 2);
      }
      for (int j = nsl >= 2 ? nsl - 2 : 0; j < nsl && ok; ++j) load_w2(j);
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
    for (int64_t it = blockIdx.x, i = 0; it < items && ok; it += gridDim.x, ++i) {
      for (int js = 0; js < nsl && ok; ++js) {
        const int64_t g = i * nsl + js;
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
      for (int j = nsl >= 2 ? nsl - 2 : 0; j < nsl && tail_ok; ++j)
        tail_ok = do_o(i * nsl + j, j, i);
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
    for (int64_t it = blockIdx.x, i = 0; it < items && ok; it += gridDim.x, ++i) {
      const int64_t qt = it / H;
      const int head = (int)(it % H);
      const int64_t qi = qt * BM + row;
      for (int js = 0; js < nsl && ok; ++js) {
        const int64_t g = i * nsl + js;
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
  __nv_bfloat16 *b1, *b3, *b2t, *U, *DH1, *DH3;
  float *partials, *scratch;
};

TcWs carve(const Problem& p, void* ws, int S) {
  TcWs w;
  char* c = static_cast<char*>(ws);
  const size_t wsz = (size_t)p.H * p.hid * p.d;
  w.b1 = reinterpret_cast<__nv_bfloat16*>(c);
  w.b3 = w.b1 + wsz;
  w.b2t = w.b3 + wsz;
  c += align_up(3 * wsz * 2, 1024);
  const size_t inter = (size_t)p.H * p.n * p.hid;
  w.U = reinterpret_cast<__nv_bfloat16*>(c);
  c += align_up(inter * 2, 1024);
  w.DH1 = reinterpret_cast<__nv_bfloat16*>(c);
  c += align_up(inter * 2, 1024);
  w.DH3 = reinterpret_cast<__nv_bfloat16*>(c);
  c += align_up(inter * 2, 1024);
  w.partials = reinterpret_cast<float*>(c);
  c += align_up((size_t)S * p.H * 3 * p.hid * p.d * 4, 1024);
  w.scratch = reinterpret_cast<float*>(c);
  return w;
}

int grad_ctas_per_split(const Problem& p) {
  const int tiles = p.hid / BM;
  return p.H * tiles + p.H * ((tiles + 1) / 2);
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
  const size_t wsz = (size_t)p.H * p.hid * p.d;
  if (p.n > 0) {
    {
      TraceScope ts("tc_convert_weights", st);
      const int cb = p.H * (p.hid / 32) * (p.d / 32);
      convert_weights_kernel<<<cb, 256, 0, st>>>(p.H, p.d, p.hid, W1, W2, W3, w.b1, w.b3, w.b2t);
    }
    CUtensorMap mK, mV, mW1, mW3, mW2t, mDH1, mDH3, mU, mKg, mVg, mUs, mD1s, mD3s;
    const uint64_t ld = (uint64_t)p.H * D;
    {
      // {64 d, tokens, d-chunks of all heads}: fb boxes are FB::CPS chunks of 128
      // tokens, grad boxes all D/64 chunks of one head for 64 tokens.
      const uint64_t dims3[3] = {(uint64_t)CH, (uint64_t)p.n, ld / CH};
      const uint64_t str3[2] = {ld * 2, CH * 2};
      const uint32_t box3[3] = {CH, BM, (uint32_t)FB<D>::CPS};
      const uint32_t boxg[3] = {CH, TK, (uint32_t)(D / CH)};
      if (!make_map(&mK, K, 3, dims3, str3, box3) || !make_map(&mV, V, 3, dims3, str3, box3) ||
          !make_map(&mKg, K, 3, dims3, str3, boxg) || !make_map(&mVg, V, 3, dims3, str3, boxg))
        return cudaErrorInvalidValue;
    }
    {
      const uint64_t dims[2] = {(uint64_t)D, (uint64_t)p.H * p.hid}, str[1] = {(uint64_t)D * 2};
      const uint32_t box[2] = {CH, HS};
      if (!make_map(&mW1, w.b1, 2, dims, str, box) || !make_map(&mW3, w.b3, 2, dims, str, box) ||
          !make_map(&mW2t, w.b2t, 2, dims, str, box))
        return cudaErrorInvalidValue;
    }
    {
      // stores (fb): {hidden, tokens, heads}, box [128 tokens x 64 hidden]
      const uint64_t dims[3] = {(uint64_t)p.hid, (uint64_t)p.n, (uint64_t)p.H};
      const uint64_t str[2] = {(uint64_t)p.hid * 2, (uint64_t)p.n * p.hid * 2};
      const uint32_t boxs[3] = {CH, BM, 1};
      // loads (grad): {64 hidden, tokens, hidden chunks, heads}, box = 2 chunks x 64 tokens
      const uint64_t dims4[4] = {(uint64_t)CH, (uint64_t)p.n, (uint64_t)(p.hid / CH),
                                 (uint64_t)p.H};
      const uint64_t str4[3] = {(uint64_t)p.hid * 2, CH * 2, (uint64_t)p.n * p.hid * 2};
      const uint32_t box4[4] = {CH, TK, 2, 1};
      if (!make_map(&mDH1, w.DH1, 4, dims4, str4, box4) ||
          !make_map(&mDH3, w.DH3, 4, dims4, str4, box4) ||
          !make_map(&mU, w.U, 4, dims4, str4, box4) || !make_map(&mUs, w.U, 3, dims, str, boxs) ||
          !make_map(&mD1s, w.DH1, 3, dims, str, boxs) || !make_map(&mD3s, w.DH3, 3, dims, str, boxs))
        return cudaErrorInvalidValue;
    }
    // fb: (head, slice) groups x token-range replicas, see fb_item_range.
    const int sms = num_sms();
    const int groups = p.H * (p.hid / HS);
    const int reps = groups <= sms ? sms / groups : 0;
    const int grid_fb = reps > 0 ? groups * reps : sms;
    cudaError_t e = ensure_smem_attr(fb_kernel<D>, FB<D>::SMEM);
    if (e != cudaSuccess) return e;
    {
      TraceScope ts("tc_fwd_bwd", st);
      fb_kernel<D><<<grid_fb, FB<D>::THREADS, FB<D>::SMEM, st>>>(
          mK, mV, mW1, mW3, mW2t, mUs, mD1s, mD3s, eta, p.n, p.H, p.hid, reps, err);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int tiles = p.hid / BM;
    const int k0 = p.H * tiles, k1 = p.H * ((tiles + 1) / 2);
    e = ensure_smem_attr(grad_kernel<D>, GR<D>::SMEM);
    if (e != cudaSuccess) return e;
    {
      TraceScope ts("tc_grad", st);
      grad_kernel<D><<<sp.S * (k0 + k1), GR<D>::THREADS, GR<D>::SMEM, st>>>(
          mDH1, mDH3, mU, mKg, mVg, p.n, p.H, p.hid, sp.chunk, k0, k1, w.partials, err);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  } else {
    cudaMemsetAsync(w.partials, 0, (size_t)sp.S * p.H * 3 * p.hid * p.d * 4, st);
  }
  if (partial_out != nullptr)
    return sum_splits(sp.S, (size_t)p.H * 3 * p.hid * p.d, w.partials, partial_out, st);
  return ns_then_renorm(p, sp.S, w.partials, static_cast<char*>(ws) + tc_main_bytes(p), true, W1,
                        W2, W3, W1o, W2o, W3o, shadow, w.scratch, st);
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
  const int sms = num_sms();
  const unsigned grid = (unsigned)(items < sms ? items : sms);
  {
    TraceScope ts("tc_apply", st);
    apply_kernel<D><<<grid, AP<D>::THREADS, AP<D>::SMEM, st>>>(
        mQ, mW13, mW2, p.n, p.H, p.hid, static_cast<__nv_bfloat16*>(O), err);
  }
  return cudaGetLastError();
}

}  // namespace

SplitPlan tc_split_plan(const Problem& p) {
  const int per = grad_ctas_per_split(p);
  int S = 148 / per;
  if (S < 1) S = 1;
  // at least 512 tokens per split: below that the fp32 partials (6.3 MB per
  // split for 4 heads of d 256) cost more than the parallelism gains
  const int64_t max_s = (p.n + 511) / 512;
  if (S > max_s) S = (int)(max_s < 1 ? 1 : max_s);
  int64_t chunk = (p.n + S - 1) / S;
  chunk = (chunk + TK - 1) / TK * TK;
  if (chunk < TK) chunk = TK;
  return {S, chunk};
}

size_t tc_main_bytes(const Problem& p) {
  const SplitPlan sp = tc_split_plan(p);
  const size_t wsz = (size_t)p.H * p.hid * p.d;
  const size_t inter = (size_t)p.H * p.n * p.hid;
  size_t b = align_up(3 * wsz * 2, 1024);
  b += 3 * align_up(inter * 2, 1024);
  b += align_up((size_t)sp.S * p.H * 3 * p.hid * p.d * 4, 1024);
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
