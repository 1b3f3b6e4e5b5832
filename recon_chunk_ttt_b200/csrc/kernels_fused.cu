// Fused TTT update on sm_100a: forward, backward and token-reduction GEMMs of
// one gradient step in one clustered kernel, with the η-scaled intermediates
// kept on chip (kimjy99 ZipMap review, section 2 "Feature Backbone", Eq. 1-3):
//
//   h1 = W1 k, h3 = W3 k, u = SiLU(h1) ⊙ h3, du = -W2^T v,
//   dh3 = du ⊙ SiLU(h1), dh1 = du ⊙ h3 ⊙ SiLU'(h1),
//   G1 = Σ_i η_i dh1_i k_i^T,  G3 = Σ_i η_i dh3_i k_i^T,  P2 = Σ_i η_i u_i v_i^T (= -G2^T).
//
// A cluster of three CTAs (one per SM) owns one head, one group of 128 hidden
// units and one contiguous token range (a split).  Per 128-token tile:
//   ranks 0 and 1 ("F", hidden units 64r .. 64r+63 of the group)
//     F    = K [W1s; W3s]^T            M = 128 tokens, N = 128, into TMEM (2 buffers)
//     epilogue: with du from rank 2, η·u (bf16) goes to rank 2, η·dh1 and η·dh3
//     (bf16) to this CTA's shared memory
//     G13 += [η·dh1 | η·dh3]^T K       M = 128 (64 dh1 rows, 64 dh3 rows), N = d, in TMEM
//   rank 2 ("D", all 128 hidden units of the group)
//     DU   = V W2s^T                   M = 128 tokens, N = 128, into TMEM (2 buffers)
//     epilogue: du (bf16) to ranks 0 and 1
//     P2  += (η·u)^T V                 M = 128 hidden, N = d, in TMEM
// The forward and the gradient MMAs have an issuing thread each, so the
// wait of one for its operands (the forward tile, or the epilogue's η-scaled
// block and the gradient ring) does not hold up the other; the forward MMAs
// run ahead, and a tile's epilogue and exchanges overlap the next tile's
// forward MMAs.  At the end
// each CTA writes its slice of the split's fp32 partial ([S][H][3][hid*d],
// blocks G1, G3, P2 as [d][hid]); a fixed-order reduction over the splits
// follows in another kernel, so results are bitwise reproducible.
//
// The exchanges are bulk copies (cp.async.bulk shared::cta -> shared::cluster)
// from a staging buffer of the sender into the receiver's operand buffer,
// completing on the receiver's mbarrier; the receiver frees the buffer by a
// remote mbarrier arrive (rank 2's MMA by a tcgen05.commit to ranks 0 and 1).
// No TMA load uses multicast.  Every wait is bounded; a CTA that gives up sets
// the abort flag of all three CTAs and the device error word.

#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc_util.cuh"

namespace ttt {

namespace {

template <int D>
struct FU {
  static constexpr int NCH = D / CH;            // 64-wide d chunks
  static constexpr int GH = 128;                // hidden units per cluster
  static constexpr int FH = 64;                 // hidden units per F CTA
  // Ring shapes (measured at scene700 size, with separate forward and
  // gradient issuers): the forward ring holds one k (or v) tile as two 32 KB
  // boxes (half of d each), so the next tile's first half loads while this
  // tile's second half is multiplied (2.5 % faster than one 64 KB box, 3-4 %
  // faster than four 16 KB boxes); the gradient ring two 16 KB stages (one
  // 32 KB or four 8 KB stages: 3-4 % slower).
  static constexpr int TKG = 32;                // tokens per gradient stage
  static constexpr int NKF = 2;                 // forward ring stages
  static constexpr int NKG = 2;                 // gradient ring: [TKG tokens x d] stages
  static constexpr int CPS_ = 2;                // d-chunks per forward stage (one TMA box)
  static constexpr int CPS = CPS_ < NCH ? CPS_ : NCH;
  static_assert(NCH % CPS == 0, "chunks per stage");
  static constexpr int CHUNK = BM * 128;        // 16 KB: 128 rows x 64 bf16
  static constexpr int KF_STAGE = CPS * CHUNK;
  static constexpr int KG_STAGE = TKG * D * 2;
  static constexpr int XB = BM * 128;           // exchange block: 128 tokens x 64 bf16 (16 KB)
  static constexpr int W2BLK = D * 128;         // D: one block of 64 hidden units x d rows
  // F: NCH K-major chunks of [128 rows (64 of W1, 64 of W3) x 64 d];
  // D: 2 MN-major blocks of [d rows x 64 hidden units] of W2 (same bytes)
  static constexpr int OFF_W = 0;
  static constexpr int OFF_KF = OFF_W + NCH * CHUNK;
  static constexpr int OFF_KG = OFF_KF + NKF * KF_STAGE;
  static constexpr int OFF_GA = OFF_KG + NKG * KG_STAGE;  // A of the gradient MMA: 2 blocks
  static constexpr int OFF_EX = OFF_GA + 2 * XB;          // F: du in | η·u out; D: du out x 2
  static constexpr int OFF_BAR = OFF_EX + 2 * XB;
  static constexpr int NBAR = 2 * NKF + 2 * NKG + 16;
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;  // + tmem slot, abort, alignment
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static constexpr int EPI_WARPS = 16;          // four per TMEM lane quadrant
  static constexpr int EPI_THREADS = 32 * EPI_WARPS;
  // kf producer, forward MMA issuer, kg producer, epilogue warps, one
  // signalling warp, gradient MMA issuer
  static constexpr int THREADS = 96 + EPI_THREADS + 64;
  static constexpr int SIGNAL_WARP = 3 + EPI_WARPS;
  static constexpr int GMMA_WARP = SIGNAL_WARP + 1;   // gradient MMA issuer
  static constexpr uint32_t TMEM_COLS = 512;    // forward buffers at 0 and 128, gradient at 256
  static constexpr uint32_t TM_G = 256;
};

// Barrier slots (same offsets in every CTA of the cluster, so a multicast
// commit and the remote arrives find them).
template <int D>
struct Bars {
  uint64_t* base;
  __device__ uint64_t* kf_full(int s) { return base + s; }
  __device__ uint64_t* kf_empty(int s) { return base + FU<D>::NKF + s; }
  __device__ uint64_t* kg_full(int s) { return base + 2 * FU<D>::NKF + s; }
  __device__ uint64_t* kg_empty(int s) { return base + 2 * FU<D>::NKF + FU<D>::NKG + s; }
  __device__ uint64_t* x(int i) { return base + 2 * FU<D>::NKF + 2 * FU<D>::NKG + i; }
  __device__ uint64_t* w_full() { return x(0); }
  __device__ uint64_t* acc_full(int b) { return x(1 + b); }
  __device__ uint64_t* acc_empty(int b) { return x(3 + b); }
  __device__ uint64_t* ga_full() { return x(5); }     // F: η·dh1|η·dh3 written; D: η·u arrived
  __device__ uint64_t* ga_empty() { return x(6); }    // F: G13 of the tile done
  __device__ uint64_t* g_full() { return x(7); }      // last gradient MMA done
  __device__ uint64_t* done() { return x(8); }
  __device__ uint64_t* au_empty() { return x(9); }    // F: rank 2's P2 read the η·u block
  __device__ uint64_t* du_full() { return x(10); }    // F: du of the tile arrived
  __device__ uint64_t* du_empty(int f) { return x(11 + f); }  // D: rank f read its du
  __device__ uint64_t* du_read() { return x(13); }    // F: every epilogue warp read du
  __device__ uint64_t* g_empty() { return x(14); }    // gradient accumulator drained
  __device__ uint64_t* done_g() { return x(15); }
};

// Give up: device error word, and the abort flag of every CTA of the cluster.
__device__ __forceinline__ void cluster_abort(volatile int* abort, int* err, int reason) {
  atomicExch(err, reason);
  const uint32_t a = smem_u32(const_cast<int*>(abort));
#pragma unroll
  for (uint32_t r = 0; r < 3; ++r)
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(mapa_shared(a, r)), "r"(1) : "memory");
}

// Bounded wait on a local mbarrier.  On a time-out the reason goes to the
// device error word and the abort flag of every CTA of the cluster is set, so
// the others leave their waits at once.  kCluster: arrivals may come from
// other CTAs (acquire at cluster scope).
template <bool kCluster>
__device__ __forceinline__ bool cwait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                      int* err, int reason) {
  auto probe = [&]() { return kCluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity); };
  if (probe()) return true;
  const long long t0 = clock64();
  while (true) {
    if (probe()) return true;
    if (*abort) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      cluster_abort(abort, err, reason);
      return false;
    }
  }
}

// Final waits before the CTA may leave: bounded, not cut short by the abort
// flag, so no asynchronous arrival can still be on its way here.
__device__ __forceinline__ void final_wait(uint64_t* bar, uint32_t parity, int* err) {
  volatile int never = 0;
  cwait<true>(bar, parity, &never, err, kErrWaitFinal);
}

// Work split.  Clusters come in sets of `groups` (the hidden units of a head
// in groups of 128), cluster `grp` of a set taking hidden group grp.  The
// head-major tile space (H heads x ntg tiles of 128 tokens) is cut into NS
// equal contiguous ranges, one per set, so the clusters of a set walk the
// same k/v tiles at the same pace (one read from HBM, the rest from L2).  The
// part of a range inside one head is a segment; a range holds one segment, or
// the end of one head and the start of the next.  Piece p of a (head, group)
// is the segment of the p-th set whose range meets the head, and its gradient
// goes to partial slot p; slots a head has no piece for are written as zeros
// by the set holding its last piece.  All of it is a function of (n, shape,
// NS), so the split sums are fixed.
// For small n (few tiles per head) a range that crosses a head would pay a
// second weight staging and gradient drain on a short critical path, so the
// sets are instead aligned to heads: SPH sets per head, each a contiguous
// part of one head's tiles (one segment, piece = part).
struct Seg {
  int head, grp;     // group of the segment
  int64_t ta;        // first tile of the segment within its group
  int nts;           // tiles in the segment
  int base;          // index of its first tile among the cluster's tiles
  int p;             // piece (partial slot) of the group
  bool last;         // the group's last piece
};
__host__ __device__ __forceinline__ int64_t range_lo(int c, int NC, int64_t T) {
  return (int64_t)c * T / NC;
}
// Start of set c's range when the sets are aligned to heads, SPH per head.
__host__ __device__ __forceinline__ int64_t aligned_lo(int c, int SPH, int64_t ntg) {
  return (int64_t)(c / SPH) * ntg + (int64_t)(c % SPH) * ntg / SPH;
}
// The set whose range holds tile index x of the head-major space.
__host__ __device__ __forceinline__ int cluster_of(int64_t x, int NC, int64_t T) {
  int c = (int)(x * NC / T);
  while (c > 0 && range_lo(c, NC, T) > x) --c;
  while (c + 1 < NC && range_lo(c + 1, NC, T) <= x) ++c;
  return c;
}
__device__ __forceinline__ Seg make_seg(int c, int NC, int SPH, int64_t T, int64_t ntg, int grp,
                                        int sg) {
  if (SPH > 0) {
    // head-aligned: one segment, piece = part of the head
    const int64_t a = aligned_lo(c, SPH, ntg), b = aligned_lo(c + 1, SPH, ntg);
    Seg s;
    s.head = c / SPH;
    s.grp = grp;
    s.ta = a - (int64_t)s.head * ntg;
    s.nts = (int)(b - a);
    s.base = 0;
    s.p = c % SPH;
    s.last = s.p == SPH - 1;
    return s;
  }
  const int64_t lo = range_lo(c, NC, T), hi = range_lo(c + 1, NC, T);
  const int64_t g = lo / ntg + sg;  // head
  const int64_t a = g * ntg > lo ? g * ntg : lo;
  const int64_t b = (g + 1) * ntg < hi ? (g + 1) * ntg : hi;
  Seg s;
  s.head = (int)g;
  s.grp = grp;
  s.ta = a - g * ntg;
  s.nts = (int)(b - a);
  s.base = (int)(a - lo);
  s.p = c - cluster_of(g * ntg, NC, T);
  s.last = c == cluster_of((g + 1) * ntg - 1, NC, T);
  return s;
}

template <int D>
__global__ void __launch_bounds__(FU<D>::THREADS, 1)
    fused_update_kernel(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
                        const __grid_constant__ CUtensorMap mKg,
                        const __grid_constant__ CUtensorMap mVg,
                        const float* __restrict__ W1, const float* __restrict__ W2,
                        const float* __restrict__ W3, const float* __restrict__ eta,
                        int64_t n, int H, int hid, int NS, int SPH, int S,
                        float* __restrict__ partials, int* err) {
  using L = FU<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  Bars<D> bar{reinterpret_cast<uint64_t*>(smem + L::OFF_BAR)};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_BAR + L::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int rank = (int)cluster_ctarank();
  const bool isF = rank < 2;
  const int groups = hid / L::GH;
  const int set = blockIdx.x / 3 / groups, grp = blockIdx.x / 3 % groups;
  const int64_t ntg = (n + BM - 1) / BM;
  const int64_t T = (int64_t)H * ntg;
  const int64_t lo = SPH > 0 ? aligned_lo(set, SPH, ntg) : range_lo(set, NS, T);
  const int64_t hi = SPH > 0 ? aligned_lo(set + 1, SPH, ntg) : range_lo(set + 1, NS, T);
  const int NT = (int)(hi - lo);                        // tiles of this cluster
  const int nseg = NT <= 0 ? 0 : SPH > 0 ? 1 : (int)((hi - 1) / ntg - lo / ntg + 1);
  auto seg = [&](int sg) { return make_seg(set, NS, SPH, T, ntg, grp, sg); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < L::NKF; ++i) {
      mbar_init(bar.kf_full(i), 1);
      mbar_init(bar.kf_empty(i), 1);
    }
    for (int i = 0; i < L::NKG; ++i) {
      mbar_init(bar.kg_full(i), 1);
      mbar_init(bar.kg_empty(i), 1);
    }
    mbar_init(bar.w_full(), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar.acc_full(b), 1);
      mbar_init(bar.acc_empty(b), L::EPI_WARPS);
    }
    mbar_init(bar.ga_full(), 1);
    mbar_init(bar.ga_empty(), 1);
    mbar_init(bar.g_full(), 1);
    mbar_init(bar.g_empty(), 1);
    mbar_init(bar.done(), 1);
    mbar_init(bar.done_g(), 1);
    mbar_init(bar.au_empty(), 1);
    mbar_init(bar.du_full(), 1);
    mbar_init(bar.du_empty(0), 1);
    mbar_init(bar.du_empty(1), 1);
    mbar_init(bar.du_read(), L::EPI_WARPS);
    *abort_flag = 0;
    fence_mbar_init();
    // Receivers arm their own exchange barriers (the senders' bulk copies
    // only complete bytes): F expects its du block, D both η·u blocks.
    if (NT > 0) {
      if (isF)
        mbar_arrive_expect_tx(bar.du_full(), L::XB);
      else
        mbar_arrive_expect_tx(bar.ga_full(), 2 * L::XB);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  // every CTA's barriers exist before any remote arrive or copy targets them
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_launch();
  grid_dep_wait();

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ forward ring
    const CUtensorMap* m = isF ? &mK : &mV;
    tma_prefetch_desc(m);
    int stage = 0;
    uint32_t phase = 0;
    int64_t issued = 0;
    bool ok = true;
    for (int sg = 0; sg < nseg && ok; ++sg) {
      const Seg S_ = seg(sg);
      for (int i = 0; i < S_.nts && ok; ++i) {
        const int y = (int)((S_.ta + i) * BM);
        for (int c = 0; c < L::NCH; c += L::CPS) {
          if (!cwait<false>(bar.kf_empty(stage), phase ^ 1, abort_flag, err, kErrWaitEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar.kf_full(stage), L::KF_STAGE);
          TTT_DCHECK((int64_t)y < n && S_.head * L::NCH + c + L::CPS <= H * L::NCH, err,
                     kErrCheckTma);
          // one box: CPS chunks of [128 tokens x 64 d]
          tma_load_3d(smem + L::OFF_KF + stage * L::KF_STAGE, m, bar.kf_full(stage), 0, y,
                      S_.head * L::NCH + c);
          ++issued;
          if (++stage == L::NKF) { stage = 0; phase ^= 1; }
        }
      }
    }
    drain_ring(bar.kf_full(0), L::NKF, issued, err);
  } else if (warp == 2 && lane == 0) {
    // ------------------------------------------------ gradient ring
    const CUtensorMap* m = isF ? &mKg : &mVg;
    tma_prefetch_desc(m);
    int stage = 0;
    uint32_t phase = 0;
    int64_t issued = 0;
    bool ok = true;
    for (int sg = 0; sg < nseg && ok; ++sg) {
      const Seg S_ = seg(sg);
      for (int i = 0; i < S_.nts && ok; ++i) {
        const int y = (int)((S_.ta + i) * BM);
        for (int st = 0; st < BM / L::TKG; ++st) {
          if (!cwait<false>(bar.kg_empty(stage), phase ^ 1, abort_flag, err, kErrWaitEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar.kg_full(stage), L::KG_STAGE);
          TTT_DCHECK((int64_t)(y + st * L::TKG) < n + BM && S_.head < H, err, kErrCheckTma);
          // one box: NCH d-chunks x [TKG tokens x 64 d]
          tma_load_3d(smem + L::OFF_KG + stage * L::KG_STAGE, m, bar.kg_full(stage), 0,
                      y + st * L::TKG, S_.head * L::NCH);
          ++issued;
          if (++stage == L::NKG) { stage = 0; phase ^= 1; }
        }
      }
    }
    drain_ring(bar.kg_full(0), L::NKG, issued, err);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------ forward MMA issuer
    // F: B = [W1s; W3s] rows, K-major; D: B = W2 columns of the group,
    // MN-major (two blocks of 64 hidden units x d rows)
    const uint32_t idF = idesc_bf16_f32(BM, 128, false, !isF);
    const uint32_t sbase = smem_u32(smem);
    int fs = 0;
    uint32_t fph = 0;
    bool ok = true;
    for (int sg = 0; sg < nseg && ok; ++sg) {
      const Seg S_ = seg(sg);
      // this segment's weights are staged
      if (!cwait<false>(bar.w_full(), (uint32_t)(sg & 1), abort_flag, err, kErrWaitFull)) {
        ok = false;
        break;
      }
      for (int i = 0; i < S_.nts && ok; ++i) {
        const int gi = S_.base + i;
        const int b = gi & 1;
        if (!cwait<false>(bar.acc_empty(b), ((gi >> 1) & 1) ^ 1, abort_flag, err,
                          kErrWaitAccFree)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dF = tmem + b * 128;
        for (int c0 = 0; c0 < L::NCH && ok; c0 += L::CPS) {
          if (!cwait<false>(bar.kf_full(fs), fph, abort_flag, err, kErrWaitFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int cc = 0; cc < L::CPS; ++cc) {
            const int c = c0 + cc;
            const uint32_t a = sbase + L::OFF_KF + fs * L::KF_STAGE + cc * L::CHUNK;
#pragma unroll
            for (int kk = 0; kk < CH / 16; ++kk) {
              const uint64_t db =
                  isF ? sdesc_sw128(sbase + L::OFF_W + c * L::CHUNK + kk * KSTEP_BYTES, 16, 1024)
                      : sdesc_sw128(sbase + L::OFF_W + (c * CH + kk * 16) * 128, L::W2BLK, 1024);
              umma_bf16(dF, sdesc_sw128(a + kk * KSTEP_BYTES, 16, 1024), db, idF,
                        (c | kk) != 0);
            }
          }
          umma_commit(bar.kf_empty(fs));
          if (++fs == L::NKF) { fs = 0; fph ^= 1; }
        }
        if (!ok) break;
        umma_commit(bar.acc_full(b));
      }
    }
    umma_commit(bar.done());
    volatile int never = 0;
    mbar_wait(bar.done(), 0, &never, err, kErrWaitFinal);
  } else if (warp == L::GMMA_WARP) {
    // ------------------------------------------------ gradient MMA issuer
    // (lane 0; the other lanes of the warp have no role)
   if (lane == 0) {
    // Its own thread, so that its operand waits (the epilogue's η-scaled
    // block, the gradient ring) overlap the forward issuer's.
    const uint32_t idG = idesc_bf16_f32(BM, D, true, true);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t ga = sbase + L::OFF_GA;
    int gs = 0;
    uint32_t gph = 0;
    bool ok = true;
    for (int sg = 0; sg < nseg && ok; ++sg) {
      const Seg S_ = seg(sg);
      // the previous segment's gradient is drained
      if (sg >= 1 && !cwait<false>(bar.g_empty(), (uint32_t)((sg - 1) & 1), abort_flag, err,
                                   kErrWaitAccFree)) {
        ok = false;
        break;
      }
      for (int i = 0; i < S_.nts && ok; ++i) {
        const int j = S_.base + i;
        const bool got =
            isF ? cwait<false>(bar.ga_full(), (uint32_t)(j & 1), abort_flag, err, kErrWaitOperand)
                : cwait<true>(bar.ga_full(), (uint32_t)(j & 1), abort_flag, err, kErrWaitOperand);
        if (!got) { ok = false; break; }
        if (!isF && j + 1 < NT) mbar_arrive_expect_tx(bar.ga_full(), 2 * L::XB);
        tc_fence_after();
        for (int st = 0; st < BM / L::TKG && ok; ++st) {
          if (!cwait<false>(bar.kg_full(gs), gph, abort_flag, err, kErrWaitFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kg = sbase + L::OFF_KG + gs * L::KG_STAGE;
#pragma unroll
          for (int kk = 0; kk < L::TKG / 16; ++kk) {
            // A: MN-major, 2 blocks of 64 rows (LBO), 16 tokens per K step;
            // B: MN-major, NCH blocks of 64 d (LBO = TKG rows x 128 B)
            const uint64_t da = sdesc_sw128(ga + (st * L::TKG + kk * 16) * 128, L::XB, 1024);
            const uint64_t db = sdesc_sw128(kg + kk * 16 * 128, L::TKG * 128, 1024);
            umma_bf16(tmem + L::TM_G, da, db, idG, (i | st | kk) != 0);
          }
          umma_commit(bar.kg_empty(gs));
          if (++gs == L::NKG) { gs = 0; gph ^= 1; }
        }
        if (!ok) break;
        if (isF)
          umma_commit(bar.ga_empty());
        else
          umma_commit_cluster(bar.au_empty(), (uint16_t)0x3);  // ranks 0 and 1 may refill
      }
      if (ok) umma_commit(bar.g_full());
    }
    umma_commit(bar.done_g());
    volatile int never = 0;
    mbar_wait(bar.done_g(), 0, &never, err, kErrWaitFinal);
   }
  } else if (warp == L::SIGNAL_WARP) {
    // ------------------------------------------------ F: du consumed -> rank 2
    // A remote arrive with cluster-scope release costs about a microsecond on
    // the issuing thread; this warp pays it so the epilogue does not.
    if (isF && lane == 0) {
      const uint32_t c_du_empty = mapa_shared(smem_u32(bar.du_empty(rank)), 2);
      for (int gi = 0; gi < NT; ++gi) {
        if (!cwait<false>(bar.du_read(), (uint32_t)(gi & 1), abort_flag, err, kErrWaitOperand))
          break;
        mbar_arrive_remote(c_du_empty);
      }
    }
  } else if (warp >= 3) {
    // ------------------------------------------------ epilogue
    const int q = warp & 3;              // TMEM lane quadrant of this warp
    const int h = (warp - 3) >> 2;       // column quarter
    const int row = q * 32 + lane;       // token row (tiles) / accumulator row (gradient)
    const bool leader = warp == 3 && lane == 0;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const int et = threadIdx.x - 96;
    const size_t mat = (size_t)hid * D;
    uint8_t* ga = smem + L::OFF_GA;
    uint8_t* ex = smem + L::OFF_EX;
    bool ok = true;
    // remote addresses
    const uint32_t c_au_full = mapa_shared(smem_u32(bar.ga_full()), 2);
    const uint32_t c_au_dst = mapa_shared(smem_u32(ga + rank * L::XB), 2);
    const uint32_t c_du_full0 = mapa_shared(smem_u32(bar.du_full()), 0);
    const uint32_t c_du_full1 = mapa_shared(smem_u32(bar.du_full()), 1);
    const uint32_t c_du_dst0 = mapa_shared(smem_u32(ex), 0);
    const uint32_t c_du_dst1 = mapa_shared(smem_u32(ex), 1);
    uint8_t* du_in = ex;
    uint8_t* au_out = ex + L::XB;
    for (int sg = 0; sg < nseg && ok; ++sg) {
      const Seg S_ = seg(sg);
      {
        // This segment's weights, fp32 -> bf16 (round to nearest) into the
        // swizzled operand layout; 16-byte granule g of a 128-byte row r sits
        // at g ^ (r % 8).  Every MMA that read the previous weights is done
        // (the previous segment's gradient was drained after g_full).
        // Both roles stage 2 * 64 * D / 8 (F) or D * 128 / 8 (rank 2) 8-element
        // granules: the same count, NG per thread; all of a thread's loads are
        // issued before its stores so their latencies overlap.
        constexpr int NG = (L::GH * D / 8) / L::EPI_THREADS;
        static_assert(NG * L::EPI_THREADS == L::GH * D / 8, "granules per thread");
        float4 wa[NG], wb[NG];
        if (isF) {
          // rows 0..63: W1, 64..127: W3 (hidden units of this CTA); a warp
          // reads one d-row of 32 granules (D = 256) at a time
          constexpr int GPR = D / 8;  // granules per weight row
#pragma unroll
          for (int k = 0; k < NG; ++k) {
            const int x = et + k * L::EPI_THREADS;
            const int r = x / GPR, gg = x % GPR;
            const float* src = (r < L::FH ? W1 : W3) + (size_t)S_.head * mat +
                               (size_t)(S_.grp * L::GH + rank * L::FH + (r % L::FH)) * D + gg * 8;
            wa[k] = __ldg(reinterpret_cast<const float4*>(src));
            wb[k] = __ldg(reinterpret_cast<const float4*>(src + 4));
          }
#pragma unroll
          for (int k = 0; k < NG; ++k) {
            const int x = et + k * L::EPI_THREADS;
            const int r = x / GPR, gg = x % GPR, c = gg / 8, g = gg % 8;
            *reinterpret_cast<uint4*>(smem + L::OFF_W + c * L::CHUNK + r * 128 +
                                      ((g ^ (r & 7)) * 16)) =
                make_uint4(pack_bf16x2(wa[k].x, wa[k].y), pack_bf16x2(wa[k].z, wa[k].w),
                           pack_bf16x2(wb[k].x, wb[k].y), pack_bf16x2(wb[k].z, wb[k].w));
          }
        } else {
          // W2[head][c][grp*128 + j]: d-row c, hidden units j of the group, as
          // two blocks of 64 units; a half-warp reads one d-row (512 bytes)
#pragma unroll
          for (int k = 0; k < NG; ++k) {
            const int x = et + k * L::EPI_THREADS;
            const int c = x / (L::GH / 8), gg = x % (L::GH / 8);
            const float* src =
                W2 + (size_t)S_.head * mat + (size_t)c * hid + S_.grp * L::GH + gg * 8;
            wa[k] = __ldg(reinterpret_cast<const float4*>(src));
            wb[k] = __ldg(reinterpret_cast<const float4*>(src + 4));
          }
#pragma unroll
          for (int k = 0; k < NG; ++k) {
            const int x = et + k * L::EPI_THREADS;
            const int c = x / (L::GH / 8), gg = x % (L::GH / 8), blk = gg / 8, g = gg % 8;
            *reinterpret_cast<uint4*>(smem + L::OFF_W + blk * L::W2BLK + c * 128 +
                                      ((g ^ (c & 7)) * 16)) =
                make_uint4(pack_bf16x2(wa[k].x, wa[k].y), pack_bf16x2(wa[k].z, wa[k].w),
                           pack_bf16x2(wb[k].x, wb[k].y), pack_bf16x2(wb[k].z, wb[k].w));
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(1, L::EPI_THREADS);
        if (leader) mbar_arrive(bar.w_full());
      }
      if (isF) {
        // η of this thread's token row, one tile ahead (its load latency is
        // not on the per-tile path)
        auto eta_of = [&](int i) -> float {
          const int64_t tok = (S_.ta + i) * BM + row;
          return i < S_.nts && tok < n ? __ldg(&eta[tok * H + S_.head]) : 0.f;
        };
        float eta_next = eta_of(0);
        for (int i = 0; i < S_.nts; ++i) {
          const int gi = S_.base + i;  // tile index within the cluster (barrier phases)
          const int b = gi & 1;
          const float ne = -eta_next;  // -η (du = -W2^T v)
          eta_next = eta_of(i + 1);
          bool got = cwait<false>(bar.acc_full(b), (uint32_t)((gi >> 1) & 1), abort_flag, err,
                                  kErrWaitAcc);
          __syncwarp();
          if (named_bar_any(1, L::EPI_THREADS, !got)) { ok = false; break; }
          tc_fence_after();
          // h1, h3 of this row for hidden units [16h, 16h + 16) of this CTA
          uint32_t r1[16], r3[16];
          const uint32_t tl = tmem + lane_base + b * 128 + h * 16;
          tmem_ld_16x(tl, r1);
          tmem_ld_16x(tl + L::FH, r3);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar.acc_empty(b));
          // η·u needs no du: form it, keep SiLU(h1) and h3·SiLU'(h1) for later
          float sa[16], shd[16];
          uint32_t pu[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            float o_u[2];
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              const float h1 = __uint_as_float(r1[e + t]);
              const float h3 = __uint_as_float(r3[e + t]);
              const float sgm = sigmoid_fast(h1);
              const float a = h1 * sgm;                      // SiLU(h1)
              sa[e + t] = a;
              shd[e + t] = h3 * fmaf(-a, sgm, a + sgm);      // h3·SiLU'(h1), SiLU' = s + a(1 - s)
              o_u[t] = -ne * (a * h3);
            }
            pu[e / 2] = pack_bf16x2(o_u[0], o_u[1]);
          }
          // η·u to rank 2, once the previous copy has read the staging buffer
          if (leader) bulk_wait_group_read0();
          named_bar_sync(1, L::EPI_THREADS);
          {
            uint8_t* r_u = au_out + row * 128;
#pragma unroll
            for (int c = 0; c < 2; ++c)
              *reinterpret_cast<uint4*>(r_u + (((2 * h + c) ^ (row & 7)) * 16)) =
                  make_uint4(pu[4 * c], pu[4 * c + 1], pu[4 * c + 2], pu[4 * c + 3]);
          }
          fence_proxy_async_smem();
          named_bar_sync(1, L::EPI_THREADS);
          if (leader) {
            // rank 2's P2 of the previous tile has read its η·u block
            if (gi >= 1 && !cwait<true>(bar.au_empty(), (uint32_t)((gi - 1) & 1), abort_flag, err,
                                        kErrWaitOperand)) {
              ok = false;
            } else {
              bulk_copy_to_cluster(c_au_dst, au_out, L::XB, c_au_full);
              bulk_commit_group();
            }
          }
          // du of this tile from rank 2
          got = cwait<true>(bar.du_full(), (uint32_t)(gi & 1), abort_flag, err, kErrWaitOperand);
          __syncwarp();
          if (named_bar_any(1, L::EPI_THREADS, !got || !ok)) { ok = false; break; }
          // every epilogue thread is past this phase: arm the next tile's du
          if (leader && gi + 1 < NT) mbar_arrive_expect_tx(bar.du_full(), L::XB);
          uint32_t dv[8];
          {
            const uint8_t* rp = du_in + row * 128;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const uint4 t = *reinterpret_cast<const uint4*>(rp + (((2 * h + c) ^ (row & 7)) * 16));
              dv[4 * c] = t.x; dv[4 * c + 1] = t.y; dv[4 * c + 2] = t.z; dv[4 * c + 3] = t.w;
            }
          }
          uint32_t p1[8], p3[8];  // η·dh1, η·dh3 as packed bf16 pairs
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const __nv_bfloat162 d2 = *reinterpret_cast<const __nv_bfloat162*>(&dv[e / 2]);
            const float e0 = ne * __low2float(d2), e1 = ne * __high2float(d2);  // η du
            p1[e / 2] = pack_bf16x2(e0 * shd[e], e1 * shd[e + 1]);
            p3[e / 2] = pack_bf16x2(e0 * sa[e], e1 * sa[e + 1]);
          }
          // du consumed (its values are in registers): the signalling warp
          // tells rank 2, off this path
          __syncwarp();
          if (lane == 0) mbar_arrive(bar.du_read());
          // the gradient MMAs of the previous tile have read the operand buffer
          if (gi >= 1) {
            got = cwait<false>(bar.ga_empty(), (uint32_t)((gi - 1) & 1), abort_flag, err,
                               kErrWaitOperand);
            __syncwarp();
            if (named_bar_any(1, L::EPI_THREADS, !got)) { ok = false; break; }
          }
          {
            uint8_t* r_1 = ga + row * 128;
            uint8_t* r_3 = ga + L::XB + row * 128;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const int pos = ((2 * h + c) ^ (row & 7)) * 16;
              *reinterpret_cast<uint4*>(r_1 + pos) =
                  make_uint4(p1[4 * c], p1[4 * c + 1], p1[4 * c + 2], p1[4 * c + 3]);
              *reinterpret_cast<uint4*>(r_3 + pos) =
                  make_uint4(p3[4 * c], p3[4 * c + 1], p3[4 * c + 2], p3[4 * c + 3]);
            }
          }
          fence_proxy_async_smem();
          named_bar_sync(1, L::EPI_THREADS);
          if (leader) mbar_arrive(bar.ga_full());
        }
      } else {
        // rank 2: du of each tile to ranks 0 and 1
        for (int i = 0; i < S_.nts; ++i) {
          const int gi = S_.base + i;
          const int b = gi & 1;
          bool got = cwait<false>(bar.acc_full(b), (uint32_t)((gi >> 1) & 1), abort_flag, err,
                                  kErrWaitAcc);
          __syncwarp();
          if (named_bar_any(1, L::EPI_THREADS, !got)) { ok = false; break; }
          tc_fence_after();
          // DU of this row for hidden units [32h, 32h + 32) of the group: rank
          // h / 2's units [32(h % 2), 32(h % 2) + 32)
          uint32_t r0[32];
          tmem_ld_32x32(tmem + lane_base + b * 128 + h * 32, r0);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar.acc_empty(b));
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(r0[2 * e]), __uint_as_float(r0[2 * e + 1]));
          if (leader) bulk_wait_group_read0();
          named_bar_sync(1, L::EPI_THREADS);
          {
            uint8_t* rp = ex + (h >> 1) * L::XB + row * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c)
              *reinterpret_cast<uint4*>(rp + (((4 * (h & 1) + c) ^ (row & 7)) * 16)) =
                  make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          }
          fence_proxy_async_smem();
          named_bar_sync(1, L::EPI_THREADS);
          if (leader) {
            for (int f = 0; f < 2 && ok; ++f) {
              // rank f has read its previous du block
              if (gi >= 1 && !cwait<true>(bar.du_empty(f), (uint32_t)((gi - 1) & 1), abort_flag,
                                          err, kErrWaitOperand)) {
                ok = false;
                break;
              }
              bulk_copy_to_cluster(f == 0 ? c_du_dst0 : c_du_dst1, ex + f * L::XB, L::XB,
                                   f == 0 ? c_du_full0 : c_du_full1);
            }
            bulk_commit_group();
          }
          if (named_bar_any(1, L::EPI_THREADS, !ok)) { ok = false; break; }
        }
      }
      if (!ok) break;
      // ---------------------------------------------- this segment's partial
      const bool have = cwait<false>(bar.g_full(), (uint32_t)(sg & 1), abort_flag, err, kErrWaitAcc);
      __syncwarp();
      if (named_bar_any(1, L::EPI_THREADS, !have)) { ok = false; break; }
      tc_fence_after();
      // slot S_.p gets the piece; a group's last piece also zeroes the slots
      // its group has no piece for
      const int slots = S_.last ? S - S_.p : 1;
      if (isF) {
        // lanes 0..63: G1 rows, 64..127: G3 rows of this CTA's 64 hidden units.
        // Each warp's 32 rows x 16 columns pass through its own 2 KB of the
        // gradient operand buffer (idle once the gradient is complete), so
        // that a store instruction writes 64 contiguous bytes of 8 rows
        // rather than 16 bytes of 32 rows.
        const int blk = q < 2 ? 0 : 1;
        const int hrow0 = S_.grp * L::GH + rank * L::FH + (q & 1) * 32;
        TTT_DCHECK(hrow0 + 32 <= hid && S_.p + slots <= S, err, kErrCheckIndex);
        uint8_t* stg = ga + (warp - 3) * 2048;  // [32 rows][4 chunks of 16 B]
        for (int c0 = h * (D / 4); c0 < (h + 1) * (D / 4); c0 += 16) {
          uint32_t rr[16];
          tmem_ld_16x(tmem + lane_base + L::TM_G + c0, rr);
          tmem_ld_wait();
          // row `lane`: chunk j at position j ^ ((lane >> 1) & 3)
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(stg + lane * 64 + ((j ^ ((lane >> 1) & 3)) * 16)) =
                make_uint4(rr[4 * j], rr[4 * j + 1], rr[4 * j + 2], rr[4 * j + 3]);
          __syncwarp();
          const int j = lane & 3;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int r = k * 8 + (lane >> 2);
            const uint4 v =
                *reinterpret_cast<const uint4*>(stg + r * 64 + ((j ^ ((r >> 1) & 3)) * 16));
            for (int z = 0; z < slots; ++z) {
              float* P = partials + (((size_t)(S_.p + z) * H + S_.head) * 3 + blk) * mat +
                         (size_t)(hrow0 + r) * D + c0 + 4 * j;
              *reinterpret_cast<uint4*>(P) = z == 0 ? v : make_uint4(0u, 0u, 0u, 0u);
            }
          }
          __syncwarp();
        }
      } else {
        // P2 rows = hidden units of the group, stored transposed as [d][hid]
        const int j = S_.grp * L::GH + row;
        TTT_DCHECK(j < hid && S_.p + slots <= S, err, kErrCheckIndex);
        for (int c0 = h * (D / 4); c0 < (h + 1) * (D / 4); c0 += 16) {
          uint32_t rr[16];
          tmem_ld_16x(tmem + lane_base + L::TM_G + c0, rr);
          tmem_ld_wait();
          for (int z = 0; z < slots; ++z) {
            float* P = partials + (((size_t)(S_.p + z) * H + S_.head) * 3 + 2) * mat;
#pragma unroll
            for (int e = 0; e < 16; ++e)
              P[(size_t)(c0 + e) * hid + j] = z == 0 ? __uint_as_float(rr[e]) : 0.f;
          }
        }
      }
      // the gradient accumulator is free for the next segment
      tc_fence_before();
      named_bar_sync(1, L::EPI_THREADS);
      if (leader) mbar_arrive(bar.g_empty());
    }
    if (leader) {
      bulk_wait_group0();
      // the last multicast arrive from rank 2 has landed before this CTA may go
      if (isF && ok && NT > 0) final_wait(bar.au_empty(), (uint32_t)((NT - 1) & 1), err);
    }
  }
  tc_fence_before();
  __syncthreads();
  // no CTA leaves while another may still copy into or arrive on it
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

template <int D>
cudaError_t fused_update_impl(const Problem& p, const float* W1, const float* W2,
                              const float* W3, const void* K, const void* V, const float* eta,
                              int NS, int SPH, int S, float* partials, int* err,
                              cudaStream_t st) {
  using L = FU<D>;
  CUtensorMap mK, mV, mKg, mVg;
  const uint64_t ld = (uint64_t)p.H * D;
  {
    // {64 d, tokens, d-chunks of all heads}
    const uint64_t dims[3] = {(uint64_t)CH, (uint64_t)p.n, ld / CH};
    const uint64_t str[2] = {ld * 2, CH * 2};
    const uint32_t boxf[3] = {CH, BM, (uint32_t)L::CPS};
    const uint32_t boxg[3] = {CH, L::TKG, (uint32_t)L::NCH};
    if (!make_map(&mK, K, 3, dims, str, boxf) || !make_map(&mV, V, 3, dims, str, boxf) ||
        !make_map(&mKg, K, 3, dims, str, boxg) || !make_map(&mVg, V, 3, dims, str, boxg))
      return cudaErrorInvalidValue;
  }
  cudaError_t e = ensure_smem_attr(fused_update_kernel<D>, L::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(3 * NS * (p.hid / L::GH)));
  cfg.blockDim = dim3(L::THREADS);
  cfg.dynamicSmemBytes = L::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 3;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  TraceScope ts("tc_update_fused", st);
  return cudaLaunchKernelEx(&cfg, fused_update_kernel<D>, mK, mV, mKg, mVg, W1, W2, W3, eta,
                            p.n, p.H, p.hid, NS, SPH, S, partials, err);
}

}  // namespace

cudaError_t fused_update(const Problem& p, const float* W1, const float* W2, const float* W3,
                         const void* K, const void* V, const float* eta, const FusedPlan& f,
                         float* partials, int* err, cudaStream_t st) {
  if (p.d == 256)
    return fused_update_impl<256>(p, W1, W2, W3, K, V, eta, f.sets, f.sets_per_head, f.splits,
                                  partials, err, st);
  return fused_update_impl<64>(p, W1, W2, W3, K, V, eta, f.sets, f.sets_per_head, f.splits,
                               partials, err, st);
}

// 3-CTA clusters of this kernel's size that are resident at once on a B200
// (148 SMs in clusters of GPCs): 45, measured with
// cudaOccupancyMaxActiveClusters; more clusters would run in a second wave.
int fused_clusters_per_wave() { return 45; }

FusedPlan fused_plan(const Problem& p) {
  FusedPlan f{1, 0, 1};
  const int64_t ntg = (p.n + BM - 1) / BM;
  const int groups = p.hid / 128;
  const int64_t T = (int64_t)p.H * ntg;
  if (T == 0) return f;
  // Few tiles per head (up to 64: 8,192 tokens): sets aligned to heads, as
  // many per head as one wave holds, at least 4 tiles each.
  const int per_wave = fused_clusters_per_wave() / groups;
  if (ntg <= 64 && per_wave >= p.H) {
    int64_t sph = per_wave / p.H;
    if (sph > ntg / 4) sph = ntg / 4;
    if (sph < 1) sph = 1;
    f.sets_per_head = (int)sph;
    f.sets = (int)(sph * p.H);
    f.splits = (int)sph;
    return f;
  }
  // as many sets of `groups` clusters as one wave holds, at least 4 tiles
  // (512 tokens) per set: below that the 6.3 MB partials (4 heads of d 256)
  // cost more than the parallelism gains
  int64_t ns = fused_clusters_per_wave() / groups;
  if (ns > T / 4) ns = T / 4;
  if (ns < 1) ns = 1;
  f.sets = (int)ns;
  for (int64_t h = 0; h < p.H; ++h) {
    const int pieces =
        cluster_of((h + 1) * ntg - 1, f.sets, T) - cluster_of(h * ntg, f.sets, T) + 1;
    if (pieces > f.splits) f.splits = pieces;
  }
  return f;
}

}  // namespace ttt
