// fa_bwd_sm100.cu -- BF16 attention backward for sm_100a.
//
// The forward keeps only O and the per-row log-sum-exp L; the backward
// recomputes P from Q, K and L instead of reading a stored N x N matrix
// (FlashAttention blog, section 2.3; CSDN FlashAttention-1 tutorial, section
// 2).  Gradients of f = sum(O * dO):
//     P  = exp(scale * Q K^T - L)        D = rowsum(dO * O)
//     dV = P^T dO     dP = dO V^T        dS = P * (dP - D)
//     dK = scale * dS^T Q                dQ = scale * dS K
//
// Centring K.  Every row of dS sums to zero (sum_j P_ij dP_ij = D_i and
// sum_j P_ij = 1), so dQ_i = scale * sum_j dS_ij (k_j - c) for any vector c
// shared by all key rows of a head; and scale * q_i . k_j = scale * q_i .
// (k_j - c) + scale * q_i . c, where the last term is constant along a row of
// S and can be moved into L.  With c = the mean of the head's first key rows
// rounded to integers, the bf16 rounding of dS is no longer multiplied by the
// mean of K (the +8-shifted K workload makes that term 8x the rest), and K - c
// is exact in bf16 whenever k and c are within a factor of two (Sterbenz) and
// equal to K when c = 0.  So the kernels keep K - c, not K, in shared memory.
//
// Launches on the caller's stream:
//   prep   1. c per (batch, key/value head) into the workspace;
//          2. per query row: D_i, L2_i = log2e * L_i - scale * log2e * q_i . c,
//             padded to 128-row blocks, and the zeroed f32 dQ accumulator;
//   dkdv   work unit = (batch, key/value head, 128-row key block); K - c and
//          V stay in shared memory and dK, dV in TMEM for the whole loop over
//          the query heads of the group and their query blocks, so dK and dV
//          need no atomics.  Per step (key rows on the 128 TMEM lanes):
//              S^T = (K-c) Q_i^T      dP^T = V dO_i^T       (tcgen05, SMEM x SMEM)
//              P^T = exp2(S^T * scale*log2e - L2_i),  dS^T = P^T * (dP^T - D_i)
//                                                           (one thread per key row)
//              dV += P^T dO_i         dK += dS^T Q_i        (tcgen05, A from TMEM)
//              dQ_i^T = (K-c)^T dS^T                        (tcgen05, SMEM x SMEM)
//          and readout warps add dQ_i^T into the f32 accumulator with float32
//          reductions.  Q_i, dO_i and the row vectors L2_i, D_i arrive
//          through a ring of TMA copies.
//          d = 64, 128: bwd_wide_kernel, persistent (one CTA per SM taking
//          units from a counter), 128-row query blocks, one TMEM score set and
//          a two-phase elementwise stage (see its comment block).
//          d = 256: the dK and dV accumulators alone fill TMEM, so
//          bwd_kernel runs two passes over the same key blocks, dV (S^T,
//          P^T, dV) then dK and dQ, with 64-row query blocks and two TMEM
//          score sets so one block's elementwise work overlaps the next
//          block's MMAs;
//   dq     dQ = bf16(scale * accumulator).
#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "launch.h"

#ifndef BWD_PERSIST
#define BWD_PERSIST 1
#endif
#ifndef BWD_GROUP_BYTES
#define BWD_GROUP_BYTES 32e6
#endif

namespace fa {
namespace {

// bwd_kernel (d = 256, two passes) warp roles: 0-7 elementwise stage (two
// warpgroups, half of the query columns each, 32 at a time; each also reads
// out and reduces a quarter of dQ^T when a step has four 32-column chunks),
// 8-11 dQ readout, 12 TMA producer, 13 MMA issuer.  The producer and MMA roles
// run in lane 0 alone (measured ~8% faster on B200 than keeping the warp
// converged around each wait).
constexpr int kThreads = 448;
constexpr int kReadoutWarp0 = 8;
constexpr int kProducerWarp = 12;
constexpr int kMmaWarp = 13;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kCenterRows = 64;   // key rows averaged into the centring vector c

enum Mode { kDV = 1, kDKDQ = 2 };   // the dV pass, then the dK and dQ pass

// BM_ query rows per step (MMA N), NSETS_ TMEM score sets, QS_ depth of the
// Q/dO ring.  An M = 128 tcgen05 MMA takes about as long for N = 64 as for
// N = 128, but with N = 128 the scores of one step fill the TMEM left next to
// dK and dV (one set), so MMA and elementwise work cannot overlap.
template <int D_, int MODE_, int BM_, int NSETS_, int QS_>
struct BwdCfg {
  static constexpr int D = D_, MODE = MODE_;
  static constexpr int BN = 128;         // key rows per CTA (MMA M)
  static constexpr int BM = BM_;
  static constexpr int NSETS = NSETS_;
  static constexpr int QS = QS_;
  static_assert(BM == 64 || BM == 128, "query block");
  static constexpr bool HAS_DP = MODE != kDV;
  static constexpr bool HAS_DV = MODE != kDKDQ;
  static constexpr bool HAS_DK = MODE != kDV;
  static constexpr bool HAS_DQ = MODE != kDV;
  static constexpr int DCH = D / 64;     // 128-byte column chunks
  static constexpr int KV_CHUNK = BN * 128;
  static constexpr int KV_TILE = KV_CHUNK * DCH;
  static constexpr int Q_CHUNK = BM * 128;
  static constexpr int Q_TILE = Q_CHUNK * DCH;
  static constexpr int DS_CHUNK = BN * 128;    // 64 query columns of dS^T (bf16)
  static constexpr int DS_TILE = DS_CHUNK * (BM / 64);
  static constexpr int ROWVEC = BM * 4;         // bytes of one query block of L2 or D
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_TILE;   // must directly follow K (d = 64 dQ MMA)
  static constexpr int OFF_Q = OFF_V + (HAS_DP ? KV_TILE : 0);
  static constexpr int OFF_DO = OFF_Q + QS * Q_TILE;
  static constexpr int OFF_DS = OFF_DO + QS * Q_TILE;
  static constexpr int OFF_L2 = OFF_DS + (HAS_DQ ? NSETS * DS_TILE : 0);
  static constexpr int OFF_DD = OFF_L2 + QS * ROWVEC;
  // dropout keep bits of a step, [128 key rows][BM query bits], two buffers
  static constexpr int MASK_BUF = BN * BM / 8;
  static constexpr int OFF_MASK = OFF_DD + QS * ROWVEC;
  static constexpr int OFF_BAR = OFF_MASK + 2 * MASK_BUF;
  // kv_full, kc_full, q_full[QS], q_empty[QS], s_full[2], p_full[2],
  // dq_full[2], dq_empty[2], final, drain, do_full[QS], do_empty[QS],
  // acc_empty, mask_full[2], mask_empty[2]
  static constexpr int NBAR = 2 + 2 * QS + 8 + 2 + 2 * QS + 1 + 4;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  // The dynamic shared window starts 1024-byte aligned (checked at run time),
  // so no alignment slack is reserved.
  static constexpr int SMEM = OFF_MISC + 16;
  // TMEM columns (a "set" holds the scores of one step).
  //   kDV   : dV [0, 256), set x at 256 + 64x: S^T [0,64); after the
  //           elementwise stage, for query columns 32h..32h+31, P^T at
  //           [32h, 32h+16)
  //   kDKDQ : dK [0, 256), set at 256: S^T [0,64) dP^T [64,128); then dS^T
  //           at [32h+16, 32h+32), dQ^T halves [128,192) and [192,256)
  static constexpr int TM_DV = 0;
  static constexpr int TM_DK = 0;
  static constexpr int TM_SET0 = D;
  static constexpr int SET_STRIDE = MODE == kDV ? BM : 2 * BM;
  static constexpr int TM_DP = BM;                          // dP^T offset inside a set
  static constexpr int TM_DQ = 128;                         // dQ^T offset inside a set
  static constexpr int NHALF = D == 256 ? 2 : 1;            // dQ^T pieces of 128 rows of d
  static constexpr int NCH = NHALF * BM / 32;               // 32-column chunks of dQ^T
  // the readout warpgroup reads dQ^T chunks 0, 1; the elementwise warpgroups
  // chunks 2, 3 when a step has four
  static constexpr int DQ_READERS = (NHALF * BM / 32) == 4 ? 384 : 128;
  static constexpr int TM_ALLOC = 512;
  static_assert(TM_SET0 + NSETS * SET_STRIDE + (MODE == kDKDQ ? 128 : 0) <= TM_ALLOC, "TMEM");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(D == 256, "the two passes are for d = 256");
  // with two score sets, S^T(i+1) is issued before step i's gradients release
  // Q_i / dO_i, so the ring needs a second slot
  static_assert(NSETS == 1 || QS >= 2, "two score sets need two Q/dO slots");
};

struct BwdParams {
  const float *l2;         // [B*Hq][Npad]
  const float *dsum;       // [B*Hq][Npad]
  const float *cvec;       // [B*Hkv][D]
  float *dq_acc;           // [B, Hq, Nq, D]
  int *sched;              // persistent dK/dV kernel: units handed out so far (beyond the grid)
  __nv_bfloat16 *dk, *dv;  // [B, Hkv, Nk, D]
  int Hq, Hkv, Nq, Nk, npad, nqb, nkb, BHkv;
  int hg;                  // key/value heads per group of the unit order
  float scale, scale_log2;
  int causal;
  // dropout on P (wide kernel, DROP instances): keep when the Philox word is
  // >= drop_thr; dV and dP are scaled by drop_scale = 1 / (1 - p)
  uint32_t drop_thr, seed_lo, seed_hi, drop_off;
  float drop_scale;
  unsigned *err;
};

__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Add 32 columns of dQ^T (one thread = one row d of a 128-row piece of dQ^T,
// chunk ch of the step's dQ^T columns) into the f32 accumulator.
template <class C>
__device__ __forceinline__ void reduce_dq_chunk(const uint32_t (&v)[32], float *acc_row, int ch,
                                                int d_local, int nvalid) {
  const int half = (ch * 32) / C::BM;   // which 128 rows of d
  const int cq = (ch * 32) % C::BM;     // first query column of the chunk
  if (d_local >= C::D) return;          // d = 64: lanes 64..127 carry no dQ
  float *a = acc_row + half * 128 + (size_t)cq * C::D;
#pragma unroll
  for (int c = 0; c < 32; ++c)
    if (cq + c < nvalid) atomicAdd(a + (size_t)c * C::D, __uint_as_float(v[c]));
}

template <class C, bool DROP>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
               const BwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The 128-byte swizzled tiles need a 1024-byte aligned base.
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(p.err, kErrConfig);
    return;
  }
  uint8_t *smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  uint64_t *bars = (uint64_t *)(smem + C::OFF_BAR);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const int B_KV = 0, B_KC = 1, B_QFULL = 2, B_QEMPTY = 2 + C::QS, B_SFULL = 2 + 2 * C::QS,
            B_PFULL = B_SFULL + 2, B_DQFULL = B_PFULL + 2, B_DQEMPTY = B_DQFULL + 2,
            B_FINAL = B_DQEMPTY + 2, B_DRAIN = B_FINAL + 1, B_DOFULL = B_DRAIN + 1,
            B_DOEMPTY = B_DOFULL + C::QS, B_ACCEMPTY = B_DOEMPTY + C::QS,
            B_MFULL = B_ACCEMPTY + 1, B_MEMPTY = B_MFULL + 2;
  uint32_t *tmem_slot = (uint32_t *)(smem + C::OFF_MISC);
  volatile int *abort_flag = (volatile int *)(smem + C::OFF_MISC + 4);
  const float *s_l2 = (const float *)(smem + C::OFF_L2);
  const float *s_dd = (const float *)(smem + C::OFF_DD);

  const int warp = warp_id_uniform();
  const int lane = threadIdx.x & 31;

  // Work units: (batch, key/value head, key block), head by head, inside a
  // head the key blocks with the most query blocks first (causal), so a wave
  // reads the Q, dO and dQ-accumulator tiles of a few heads, which stay in
  // L2.  Persistent CTAs (one per SM when there are more units): round k
  // gives CTA c unit k G + c (k even) or k G + G - 1 - c (k odd), G =
  // gridDim.x, so each CTA keeps its TMEM and barriers and the next unit's
  // first Q/dO tiles and K/V loads overlap the current unit's last steps and
  // epilogue.  Barrier phases follow the count of units with work (uc) and
  // of steps (gs) this CTA has processed.
  const int total_units = p.nkb * p.BHkv;
  const int G = (int)gridDim.x;
  const int g = p.Hq / p.Hkv;
  struct Unit {
    int bhkv, b, hkv, kv0, i0, nq_eff, nsteps;
  };
  auto decode = [&](int u) {
    Unit U;
    const int jblk = u % p.nkb;
    U.bhkv = u / p.nkb;
    U.b = U.bhkv / p.Hkv;
    U.hkv = U.bhkv % p.Hkv;
    U.kv0 = jblk * C::BN;
    U.i0 = p.causal ? U.kv0 / C::BM : 0;   // first query block that sees this key block
    U.nq_eff = p.nqb - U.i0;
    U.nsteps = U.nq_eff > 0 ? g * U.nq_eff : 0;
    return U;
  };
  auto unit_at = [&](int k) {
    return k * G + ((k & 1) ? G - 1 - (int)blockIdx.x : (int)blockIdx.x);
  };
  auto step_head = [&](const Unit &U, int s) { return U.hkv * g + s / U.nq_eff; };
  auto step_qblk = [&](const Unit &U, int s) { return U.i0 + s % U.nq_eff; };
  // score set and its barrier phase of the gi-th step of this CTA
  auto set_of = [&](int gi) { return C::NSETS == 2 ? (gi & 1) : 0; };
  auto set_phase = [&](int gi) { return (uint32_t)((C::NSETS == 2 ? (gi >> 1) : gi) & 1); };

  if (threadIdx.x == 0) {
    mbar_init(bar(B_KV), 1);
    mbar_init(bar(B_KC), 256);
    for (int s = 0; s < C::QS; ++s) {
      mbar_init(bar(B_QFULL + s), 1);
      mbar_init(bar(B_QEMPTY + s), 1);
      mbar_init(bar(B_DOFULL + s), 1);
      mbar_init(bar(B_DOEMPTY + s), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(B_SFULL + x), 1);
      mbar_init(bar(B_PFULL + x), 256);
      mbar_init(bar(B_DQFULL + x), 1);
      mbar_init(bar(B_DQEMPTY + x), C::DQ_READERS);
    }
    mbar_init(bar(B_FINAL), 1);
    mbar_init(bar(B_DRAIN), 1);
    mbar_init(bar(B_ACCEMPTY), 256);
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(B_MFULL + x), 128);    // the mask threads wrote their rows
      mbar_init(bar(B_MEMPTY + x), 256);   // the elementwise threads read theirs
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), C::TM_ALLOC);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    if (C::HAS_DP) prefetch_tmap(&tmV);
    prefetch_tmap(&tmDO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  WaitCtx wc{p.err, abort_flag, kWaitLimitNs};

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    // The whole role runs in lane 0; the other lanes wait at the end.
    if (lane == 0) {
      int last_q[C::QS], last_do[C::QS];
      for (int s = 0; s < C::QS; ++s) last_q[s] = last_do[s] = -1;
      int kv_phase = -1;
      bool ok = true;
      int uc = 0, gs = 0;
      // Q_i and dO_i fill separate slots.  dK/dQ pass: Q_i carries the row
      // vectors L2_i, D_i (read by the elementwise stage, Q_i last read by
      // dK(i)) and dO_i is read only by dP^T(i), so dO_{i+1} can arrive as soon
      // as dP^T(i) is done and Q_{i+1} as soon as dK(i) is.  dV pass: Q_i is
      // read only by S^T(i) and the row vectors travel with dO_i (read by
      // dV(i)), so Q_{i+2} can arrive while step i's elementwise work runs.
      constexpr uint32_t ROWS_Q = C::HAS_DP ? 2 * C::ROWVEC : 0;
      constexpr uint32_t ROWS_DO = C::HAS_DP ? 0 : 2 * C::ROWVEC;
      auto load_rows = [&](const Unit &U, int i, int st, uint32_t fb) {
        const int bh = U.b * p.Hq + step_head(U, i);
        const size_t vrow = (size_t)bh * p.npad + (size_t)step_qblk(U, i) * C::BM;
        bulk_load(sbase + C::OFF_L2 + st * C::ROWVEC, p.l2 + vrow, C::ROWVEC, fb);
        bulk_load(sbase + C::OFF_DD + st * C::ROWVEC, p.dsum + vrow, C::ROWVEC, fb);
      };
      auto load_q = [&](const Unit &U, int i, int st, uint32_t ph) {
        if (!bounded_wait(bar(B_QEMPTY + st), ph ^ 1, wc)) return false;
        const int bh = U.b * p.Hq + step_head(U, i), qb = step_qblk(U, i);
        const uint32_t fb = bar(B_QFULL + st);
        mbar_arrive_expect_tx(fb, C::Q_TILE + ROWS_Q);
        for (int c = 0; c < C::DCH; ++c)
          tma_load_3d(sbase + C::OFF_Q + st * C::Q_TILE + c * C::Q_CHUNK, &tmQ, fb, c * 64,
                      qb * C::BM, bh);
        if (ROWS_Q) load_rows(U, i, st, fb);
        last_q[st] = ph;
        return true;
      };
      auto load_do = [&](const Unit &U, int i, int st, uint32_t ph) {
        if (!bounded_wait(bar(B_DOEMPTY + st), ph ^ 1, wc)) return false;
        const int bh = U.b * p.Hq + step_head(U, i), qb = step_qblk(U, i);
        const uint32_t fb = bar(B_DOFULL + st);
        mbar_arrive_expect_tx(fb, C::Q_TILE + ROWS_DO);
        for (int c = 0; c < C::DCH; ++c)
          tma_load_3d(sbase + C::OFF_DO + st * C::Q_TILE + c * C::Q_CHUNK, &tmDO, fb, c * 64,
                      qb * C::BM, bh);
        if (ROWS_DO) load_rows(U, i, st, fb);
        last_do[st] = ph;
        return true;
      };
      // step i of unit U: the slot freed first goes first (dO in the dK/dQ
      // pass, Q in the dV pass)
      auto load_step = [&](const Unit &U, int i) {
        const int gi = gs + i;
        const int st = gi % C::QS;
        const uint32_t ph = (gi / C::QS) & 1;
        if (C::HAS_DP) return load_do(U, i, st, ph) && load_q(U, i, st, ph);
        return load_q(U, i, st, ph) && load_do(U, i, st, ph);
      };
      for (int k = 0; ok && k * G < total_units; ++k) {
        const int u = unit_at(k);
        if (u >= total_units) continue;
        const Unit U = decode(u);
        if (U.nsteps == 0) continue;
        // the first ring slots of this unit, then K (and V) once the previous
        // unit's MMAs, the last readers of K and V, are done, then the rest
        const int pre = min(C::QS, U.nsteps);
        for (int i = 0; i < pre && ok; ++i) ok = load_step(U, i);
        if (ok && uc > 0) ok = bounded_wait(bar(B_FINAL), (uc - 1) & 1, wc);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(B_KV), (C::HAS_DP ? 2 : 1) * C::KV_TILE);
        for (int c = 0; c < C::DCH; ++c) {
          tma_load_3d(sbase + C::OFF_K + c * C::KV_CHUNK, &tmK, bar(B_KV), c * 64, U.kv0, U.bhkv);
          if (C::HAS_DP)
            tma_load_3d(sbase + C::OFF_V + c * C::KV_CHUNK, &tmV, bar(B_KV), c * 64, U.kv0, U.bhkv);
        }
        kv_phase = uc & 1;
        for (int i = pre; i < U.nsteps && ok; ++i) ok = load_step(U, i);
        // the next unit's K (and V) go to L2 now, so their load after this
        // unit's last MMA does not wait on DRAM
        const int un = unit_at(k + 1);
        if (ok && (k + 1) * G < total_units && un < total_units) {
          const Unit N = decode(un);
          for (int c = 0; c < C::DCH; ++c) {
            tma_prefetch_l2_3d(&tmK, c * 64, N.kv0, N.bhkv);
            if (C::HAS_DP) tma_prefetch_l2_3d(&tmV, c * 64, N.kv0, N.bhkv);
          }
        }
        gs += U.nsteps;
        ++uc;
      }
      if (!ok) {
        if (kv_phase >= 0) (void)drain_wait(bar(B_KV), kv_phase, p.err, kWaitLimitNs);
        for (int s = 0; s < C::QS; ++s) {
          if (last_q[s] >= 0) (void)drain_wait(bar(B_QFULL + s), last_q[s], p.err, kWaitLimitNs);
          if (last_do[s] >= 0) (void)drain_wait(bar(B_DOFULL + s), last_do[s], p.err, kWaitLimitNs);
        }
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t IDESC_SP = idesc_bf16(128, C::BM, 0, 0);  // S^T, dP^T: K-major A and B
    constexpr uint32_t IDESC_KV = idesc_bf16(128, C::D, 0, 1);   // dV, dK: A TMEM, B MN-major
    constexpr uint32_t IDESC_DQ = idesc_bf16(128, C::BM, 1, 1);  // dQ^T: both MN-major
    // Descriptors are built once; each MMA offsets a base descriptor.
    const uint64_t dK_km = sw128_desc(sbase + C::OFF_K, 16, 1024);        // K-c, K-major
    const uint64_t dV_km = sw128_desc(sbase + C::OFF_V, 16, 1024);        // V, K-major
    const uint64_t dK_mn = sw128_desc(sbase + C::OFF_K, C::KV_CHUNK, 1024);  // (K-c)^T, MN-major
    const uint64_t dQ_km = sw128_desc(sbase + C::OFF_Q, 16, 1024);
    const uint64_t dQ_mn = sw128_desc(sbase + C::OFF_Q, C::Q_CHUNK, 1024);
    const uint64_t dO_km = sw128_desc(sbase + C::OFF_DO, 16, 1024);
    const uint64_t dO_mn = sw128_desc(sbase + C::OFF_DO, C::Q_CHUNK, 1024);
    const uint64_t dS_mn = sw128_desc(sbase + C::OFF_DS, C::DS_CHUNK, 1024);
    auto issue_S = [&](int x, int st) {
      const uint64_t qa = desc_add(dQ_km, st * C::Q_TILE);
      const uint32_t set = tmem + C::TM_SET0 + x * C::SET_STRIDE;
#pragma unroll
      for (int kk = 0; kk < C::D / 16; ++kk) {
        const uint32_t okv = (kk >> 2) * C::KV_CHUNK + (kk & 3) * 32;
        const uint32_t oq = (kk >> 2) * C::Q_CHUNK + (kk & 3) * 32;
        mma_ss(set, desc_add(dK_km, okv), desc_add(qa, oq), IDESC_SP, kk > 0);
      }
    };
    auto issue_dP = [&](int x, int st) {
      if (!C::HAS_DP) return;
      const uint64_t da = desc_add(dO_km, st * C::Q_TILE);
      const uint32_t set = tmem + C::TM_SET0 + x * C::SET_STRIDE;
#pragma unroll
      for (int kk = 0; kk < C::D / 16; ++kk) {
        const uint32_t okv = (kk >> 2) * C::KV_CHUNK + (kk & 3) * 32;
        const uint32_t oq = (kk >> 2) * C::Q_CHUNK + (kk & 3) * 32;
        mma_ss(set + C::TM_DP, desc_add(dV_km, okv), desc_add(da, oq), IDESC_SP, kk > 0);
      }
    };
    // dV += P^T dO_i and dK += dS^T Q_i (K = BM query rows, 16 per MMA).
    // Query rows 16 kk .. 16 kk + 15 of P^T / dS^T live in the 32-column block
    // h = kk / 2 that produced them: P^T at 32 h + [0, 16), dS^T at
    // 32 h + [16, 32).
    auto issue_dvdk = [&](int x, int st, bool first) {
      const uint64_t qa = desc_add(dQ_mn, st * C::Q_TILE);
      const uint64_t da = desc_add(dO_mn, st * C::Q_TILE);
      const uint32_t set = tmem + C::TM_SET0 + x * C::SET_STRIDE;
      if (C::HAS_DV) {
#pragma unroll
        for (int kk = 0; kk < C::BM / 16; ++kk)
          mma_ts(tmem + C::TM_DV, set + (kk >> 1) * 32 + (kk & 1) * 8, desc_add(da, kk * 2048),
                 IDESC_KV, (!first) || kk > 0);
      }
      if (C::HAS_DK) {
#pragma unroll
        for (int kk = 0; kk < C::BM / 16; ++kk)
          mma_ts(tmem + C::TM_DK, set + (kk >> 1) * 32 + 16 + (kk & 1) * 8,
                 desc_add(qa, kk * 2048), IDESC_KV, (!first) || kk > 0);
      }
    };
    // dQ_i^T = A^T dS^T with K = 128 key rows (16 per MMA), N = BM query
    // columns and M = 128 rows of A^T: [(K-c)^T ; V^T] for d = 64 (the V half
    // is unused), (K-c)^T for d = 128, and the two 128-row halves of (K-c)^T
    // for d = 256.
    auto issue_dq = [&](int x) {
      const uint32_t set = tmem + C::TM_SET0 + x * C::SET_STRIDE;
      const uint64_t dsb = desc_add(dS_mn, x * C::DS_TILE);
#pragma unroll
      for (int half = 0; half < C::NHALF; ++half) {
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk)
          mma_ss(set + C::TM_DQ + half * C::BM,
                 desc_add(dK_mn, half * 2 * C::KV_CHUNK + kk * 2048), desc_add(dsb, kk * 2048),
                 IDESC_DQ, kk > 0);
      }
    };
    // S^T (and dP^T in the dK/dQ pass) of the gi-th step into score set x.
    // The caller has waited for Q; in the dV pass Q's slot is released once
    // S^T is done with it.  dO is waited for here and, in the dK/dQ pass, its
    // slot released once dP^T is done with it.
    auto issue_scores = [&](int x, int gi) {
      const int st = gi % C::QS;
      issue_S(x, st);
      if (!C::HAS_DP) mma_commit(bar(B_QEMPTY + st));
      if (C::HAS_DP) {
        if (!bounded_wait(bar(B_DOFULL + st), (gi / C::QS) & 1, wc)) return false;
        tc_fence_after();
        issue_dP(x, st);
        mma_commit(bar(B_DOEMPTY + st));
      }
      mma_commit(bar(B_SFULL + x));
      return true;
    };
    // The whole role runs in lane 0; the other lanes wait at the end.
    if (lane == 0) {
      bool ok = true;
      int uc = 0, gs = 0;
      for (int k = 0; ok && k * G < total_units; ++k) {
        const int u = unit_at(k);
        if (u >= total_units) continue;
        const Unit U = decode(u);
        const int nsteps = U.nsteps;
        if (nsteps == 0) continue;
        // this unit's K - c in place, its first Q loaded
        ok = bounded_wait(bar(B_KC), uc & 1, wc);
        if (ok) ok = bounded_wait(bar(B_QFULL + gs % C::QS), (gs / C::QS) & 1, wc);
        if (!ok) break;
        tc_fence_after();
        ok = issue_scores(set_of(gs), gs);
        for (int i = 0; i < nsteps && ok; ++i) {
          const int gi = gs + i;
          const int x = set_of(gi);
          const int st = gi % C::QS;
          if (C::NSETS == 2 && i + 1 < nsteps) {
            const int y = x ^ 1;
            if (C::HAS_DQ && gi >= 1) {
              ok = bounded_wait(bar(B_DQEMPTY + y), set_phase(gi - 1), wc);
              if (!ok) break;
            }
            const int st1 = (gi + 1) % C::QS;
            ok = bounded_wait(bar(B_QFULL + st1), ((gi + 1) / C::QS) & 1, wc);
            if (!ok) break;
            tc_fence_after();
            ok = issue_scores(y, gi + 1);
            if (!ok) break;
          }
          ok = bounded_wait(bar(B_PFULL + x), set_phase(gi), wc);
          if (!ok) break;
          if (C::HAS_DQ && C::NSETS == 1 && gi >= 1) {
            ok = bounded_wait(bar(B_DQEMPTY + x), set_phase(gi - 1), wc);
            if (!ok) break;
          }
          if (!C::HAS_DP) {
            // the dV pass reads dO_i in dV(i)
            ok = bounded_wait(bar(B_DOFULL + st), (gi / C::QS) & 1, wc);
            if (!ok) break;
          }
          // the unit's first dV/dK start the accumulators afresh: the previous
          // unit's epilogue must have read them out of TMEM
          if (i == 0 && uc > 0) {
            ok = bounded_wait(bar(B_ACCEMPTY), (uc - 1) & 1, wc);
            if (!ok) break;
          }
          tc_fence_after();
          issue_dvdk(x, st, i == 0);
          // dK/dQ pass: Q_i is done with once dK(i) has read it, and the
          // elementwise stage finished with L2_i and D_i before p_full; dQ^T(i)
          // reads K and dS^T only.  dV pass: dO_i and its row vectors likewise.
          mma_commit(bar(C::HAS_DP ? B_QEMPTY + st : B_DOEMPTY + st));
          if (C::HAS_DQ) {
            issue_dq(x);
            mma_commit(bar(B_DQFULL + x));
          }
          if (C::NSETS == 1 && i + 1 < nsteps) {
            // S^T(i+1) only overwrites P^T/dS^T, which dV/dK(i) (issued
            // earlier) consume in order; Q_{i+1} arrives while dQ^T(i) runs
            const int st1 = (gi + 1) % C::QS;
            ok = bounded_wait(bar(B_QFULL + st1), ((gi + 1) / C::QS) & 1, wc);
            if (!ok) break;
            tc_fence_after();
            ok = issue_scores(x, gi + 1);
            if (!ok) break;
          }
        }
        if (!ok) break;
        // the unit's accumulators are final once its MMAs complete; this
        // also releases K and V to the producer
        mma_commit(bar(B_FINAL));
        gs += nsteps;
        ++uc;
      }
      if (!ok) {
        mma_commit(bar(B_DRAIN));
        (void)drain_wait(bar(B_DRAIN), 0, p.err, kWaitLimitNs);
      }
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------ elementwise stage
    const int wg = warp >> 2;                      // query columns [32 wg, 32 wg + 32)
    const int r = threadIdx.x & 127;               // key row within the block = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    // warpgroup 0 writes dV, warpgroup 1 writes dK (one key row per thread)
    const bool mine = wg == 0 ? C::HAS_DV : C::HAS_DK;
    constexpr int NCB = C::BM / 64;   // 32-column blocks per warpgroup and step
    bool ok = true;
    int uc = 0, gs = 0;
    for (int k = 0; ok && k * G < total_units; ++k) {
      const int u = unit_at(k);
      if (u >= total_units) continue;
      const Unit U = decode(u);
      const int kv = U.kv0 + r;
      const bool kv_live = kv < p.Nk;
      if (U.nsteps == 0) {
        // no query row sees this key block: its gradients are zero
        if (kv_live && mine) {
          __nv_bfloat16 *dst = (wg ? p.dk : p.dv) + ((size_t)U.bhkv * p.Nk + kv) * C::D;
          for (int e = 0; e < C::D / 8; ++e) reinterpret_cast<uint4 *>(dst)[e] = make_uint4(0, 0, 0, 0);
        }
        continue;
      }
      // K row r -> K - c in place (same swizzled layout; rows past Nk were
      // zero-filled and stay zero).  Warpgroup wg takes the 64-column chunks
      // ch = wg, wg + 2, ...
      ok = warp_wait_all(bar(B_KV), uc & 1, wc);
      if (!ok) break;
      {
        const float *cv = p.cvec + (size_t)U.bhkv * C::D;
#pragma unroll 1
        for (int ch = wg; ch < C::DCH; ch += 2) {
          uint8_t *row = smem + C::OFF_K + ch * C::KV_CHUNK + r * 128;
#pragma unroll
          for (int u8 = 0; u8 < 8; ++u8) {
            const int col = ch * 64 + ((u8 ^ (r & 7)) << 3);
            const float4 c_lo = *reinterpret_cast<const float4 *>(cv + col);
            const float4 c_hi = *reinterpret_cast<const float4 *>(cv + col + 4);
            const float cc[8] = {c_lo.x, c_lo.y, c_lo.z, c_lo.w, c_hi.x, c_hi.y, c_hi.z, c_hi.w};
            uint4 v = *reinterpret_cast<const uint4 *>(row + (u8 << 4));
            uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 h2 = *reinterpret_cast<__nv_bfloat162 *>(&w[e]);
              const float2 f = __bfloat1622float2(h2);
              w[e] = kv_live ? pack_bf16x2(f.x - cc[2 * e], f.y - cc[2 * e + 1]) : 0u;
            }
            *reinterpret_cast<uint4 *>(row + (u8 << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(bar(B_KC));
      }
      for (int i = 0; i < U.nsteps && ok; ++i) {
        const int gi = gs + i;
        const int x = set_of(gi), st = gi % C::QS;
        // the row vectors L2_i, D_i come with Q_i (dK/dQ pass) or dO_i (dV pass)
        ok = warp_wait_all(bar((C::HAS_DP ? B_QFULL : B_DOFULL) + st), (gi / C::QS) & 1, wc);
        if (ok) ok = warp_wait_all(bar(B_SFULL + x), set_phase(gi), wc);
        if (!ok) break;
        tc_fence_after();
        const uint32_t set = tmem + lane_off + C::TM_SET0 + x * C::SET_STRIDE;
        // dropout: bit c of word cb = query column 32 cb + c of the step kept for
        // this key row (the Philox words the forward used, evaluated ahead by
        // warps 8-11); the dV pass stores P^T * Z, the dK / dQ pass scales the
        // kept dP^T by 1 / (1 - p)
        uint32_t keepw[NCB];
        if (DROP) {
          ok = warp_wait_all(bar(B_MFULL + (gi & 1)), (gi >> 1) & 1, wc);
          if (!ok) break;
          const uint32_t *mrow = reinterpret_cast<const uint32_t *>(
              smem + C::OFF_MASK + (gi & 1) * C::MASK_BUF + r * (C::BM / 8));
#pragma unroll
          for (int hh = 0; hh < NCB; ++hh) keepw[hh] = mrow[wg * NCB + hh];
          mbar_arrive(bar(B_MEMPTY + (gi & 1)));
        }
#pragma unroll 1
        for (int hh = 0; hh < NCB; ++hh) {
          const int cb = wg * NCB + hh;   // 32-column block of the step
          const int c0 = cb * 32;
          uint32_t sv[32], dv[32];
          tmem_ld32(set + c0, sv);
          if (C::HAS_DP) tmem_ld32(set + C::TM_DP + c0, dv);
          tmem_wait_ld();
          const float4 *l4 = reinterpret_cast<const float4 *>(s_l2 + st * C::BM + c0);
          const float4 *d4 = reinterpret_cast<const float4 *>(s_dd + st * C::BM + c0);
          const int q0 = step_qblk(U, i) * C::BM + c0;
          // causal: key kv is hidden from query q when kv > q; key rows past
          // Nk (zero-filled) are masked so they add nothing anywhere.  Query
          // rows past Nq have L2 = +inf, so their P is 0.
          const int first_vis = !kv_live ? 32 : (p.causal ? kv - q0 : 0);
          const bool unmasked = __all_sync(0xffffffffu, first_vis <= 0);
          const uint32_t keep = DROP ? keepw[hh] : 0xffffffffu;
          uint32_t pk[16], dk[16];
          auto body = [&](auto masked_tag) {
            constexpr bool MASKED = decltype(masked_tag)::value;
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) {
              const float4 lq = l4[e4];
              const float4 dq4 = C::HAS_DP ? d4[e4] : make_float4(0.f, 0.f, 0.f, 0.f);
              const float lv[4] = {lq.x, lq.y, lq.z, lq.w};
              const float dvv[4] = {dq4.x, dq4.y, dq4.z, dq4.w};
              float pr[4], ds[4];
#pragma unroll
              for (int u4 = 0; u4 < 4; ++u4) {
                const int c = 4 * e4 + u4;
                float pv = fast_exp2(fmaf(__uint_as_float(sv[c]), p.scale_log2, -lv[u4]));
                if (MASKED) pv = (c >= first_vis) ? pv : 0.f;
                const bool kept = !DROP || ((keep >> c) & 1u);
                pr[u4] = kept ? pv : 0.f;
                float dpv = __uint_as_float(dv[c]);
                if (DROP) dpv = kept ? dpv * p.drop_scale : 0.f;
                ds[u4] = C::HAS_DP ? pv * (dpv - dvv[u4]) : 0.f;
              }
              pk[2 * e4] = pack_bf16x2(pr[0], pr[1]);
              pk[2 * e4 + 1] = pack_bf16x2(pr[2], pr[3]);
              dk[2 * e4] = pack_bf16x2(ds[0], ds[1]);
              dk[2 * e4 + 1] = pack_bf16x2(ds[2], ds[3]);
            }
          };
          if (unmasked) body(std::false_type{});
          else body(std::true_type{});
          // bf16 P^T and dS^T go into the 32 S^T columns just read, so columns
          // another thread group has not read yet are never touched
          if (C::HAS_DV) tmem_st16(set + c0, pk);
          if (C::HAS_DK) tmem_st16(set + c0 + 16, dk);
          if (C::HAS_DQ) {
            // dS^T row r -> shared memory (B operand of the dQ^T MMA: 64-column
            // chunks of 128-byte swizzled rows; 16-byte unit u of row r sits
            // at unit u ^ (r % 8))
            uint8_t *dsrow = smem + C::OFF_DS + x * C::DS_TILE + (c0 >> 6) * C::DS_CHUNK + r * 128;
            const int u0 = (c0 & 63) >> 3;
#pragma unroll
            for (int c = 0; c < 4; ++c)
              *reinterpret_cast<uint4 *>(dsrow + (((u0 + c) ^ (r & 7)) << 4)) =
                  make_uint4(dk[4 * c], dk[4 * c + 1], dk[4 * c + 2], dk[4 * c + 3]);
          }
        }
        if (C::HAS_DQ) fence_proxy_async_smem();
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_PFULL + x));
        if (C::HAS_DQ && C::NCH == 4) {
          // Share of the dQ^T readout: chunk 2 + wg (the readout warpgroup takes
          // chunks 0 and 1), so every column is in registers before dQ^T's TMEM
          // columns are released, with room to spare.
          ok = warp_wait_all(bar(B_DQFULL + x), set_phase(gi), wc);
          if (!ok) break;
          tc_fence_after();
          const int ch = 2 + wg;
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + C::TM_SET0 + x * C::SET_STRIDE + C::TM_DQ + ch * 32, v);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(bar(B_DQEMPTY + x));
          const int qb0 = step_qblk(U, i) * C::BM;
          float *acc = p.dq_acc + (((size_t)(U.b * p.Hq + step_head(U, i))) * p.Nq + qb0) * C::D + r;
          reduce_dq_chunk<C>(v, acc, ch, r, min(C::BM, p.Nq - qb0));
        }
      }
      if (!ok) break;
      // ---------------------------------------------------- epilogue
      // the accumulators are released once read, before the stores complete
      ok = warp_wait_all(bar(B_FINAL), uc & 1, wc);
      if (!ok) break;
      tc_fence_after();
      if (!mine) {
        tc_fence_before();
        mbar_arrive(bar(B_ACCEMPTY));
      } else {
        const size_t rowoff = ((size_t)U.bhkv * p.Nk + (kv_live ? kv : 0)) * C::D;
        const uint32_t src = tmem + lane_off + (wg ? C::TM_DK : C::TM_DV);
        __nv_bfloat16 *dst = (wg ? p.dk : p.dv) + rowoff;
        const float mul = wg ? p.scale : (DROP ? p.drop_scale : 1.f);
#pragma unroll 1
        for (int c = 0; c < C::D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(src + c * 32, v);
          tmem_wait_ld();
          if (c == C::D / 32 - 1) {
            tc_fence_before();
            mbar_arrive(bar(B_ACCEMPTY));
          }
          uint32_t pkd[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pkd[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * mul, __uint_as_float(v[2 * e + 1]) * mul);
          if (kv_live) {
            uint4 *o = reinterpret_cast<uint4 *>(dst + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) o[e] = make_uint4(pkd[4 * e], pkd[4 * e + 1], pkd[4 * e + 2], pkd[4 * e + 3]);
          }
        }
      }
      gs += U.nsteps;
      ++uc;
    }
  } else if (warp < kProducerWarp && (C::HAS_DQ || DROP)) {
    // ---------------------------------- dQ readout and dropout mask
    const int t = threadIdx.x - 32 * kReadoutWarp0;  // TMEM lane = column d of dQ (per half)
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    static_assert(!C::HAS_DQ || C::NCH == 2 || C::NCH == 4, "dQ^T readout split");
    static_assert(!DROP || C::BM == 64, "mask threads: 32 key quads x 4 groups of 16 query columns");
    bool ok = true;
    // Dropout mask, two steps ahead of the elementwise stage: the mask cursor
    // walks the same unit sequence (step mi of the unit at turn mk; mg counts
    // the steps, the elementwise stage's gi).  Thread t evaluates the Philox
    // counters of key rows 4 kq .. 4 kq + 3 (counter word 0 = key / 4, word j
    // of the result = key row 4 kq + j) and query columns 16 qg .. 16 qg + 15.
    int mk = -1, mi = 0, mg = -1;
    bool mend = false;
    Unit mU{};
    auto madvance = [&]() {
      if (mk >= 0 && mi + 1 < mU.nsteps) {
        ++mi;
        ++mg;
        return;
      }
      for (;;) {
        ++mk;
        if (mk * G >= total_units) {
          mend = true;
          return;
        }
        const int u = unit_at(mk);
        if (u >= total_units) continue;
        mU = decode(u);
        if (mU.nsteps > 0) {
          mi = 0;
          ++mg;
          return;
        }
      }
    };
    auto gen_mask = [&]() {
      const int buf = mg & 1;
      if (!warp_wait_all(bar(B_MEMPTY + buf), ((mg >> 1) & 1) ^ 1, wc)) return false;
      const int kq = t >> 2, qg = t & 3;
      const uint32_t kc = (uint32_t)((mU.kv0 >> 2) + kq);
      const uint32_t q = (uint32_t)(step_qblk(mU, mi) * C::BM + 16 * qg);
      const uint32_t bhq = (uint32_t)(mU.b * p.Hq + step_head(mU, mi));
      uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
#pragma unroll 4
      for (int e = 0; e < 16; ++e) {
        const uint4 R = philox4x32_10(kc, q + e, bhq, p.drop_off, p.seed_lo, p.seed_hi);
        m0 |= (R.x >= p.drop_thr ? 1u : 0u) << e;
        m1 |= (R.y >= p.drop_thr ? 1u : 0u) << e;
        m2 |= (R.z >= p.drop_thr ? 1u : 0u) << e;
        m3 |= (R.w >= p.drop_thr ? 1u : 0u) << e;
      }
      // row r of the buffer: BM bits, 16-bit piece qg = columns 16 qg .. 16 qg + 15
      uint16_t *mb = reinterpret_cast<uint16_t *>(smem + C::OFF_MASK + buf * C::MASK_BUF) +
                     (4 * kq) * (C::BM / 16) + qg;
      mb[0] = (uint16_t)m0;
      mb[C::BM / 16] = (uint16_t)m1;
      mb[2 * (C::BM / 16)] = (uint16_t)m2;
      mb[3 * (C::BM / 16)] = (uint16_t)m3;
      mbar_arrive(bar(B_MFULL + buf));
      return true;
    };
    if (DROP) {
      for (int pre = 0; pre < 2 && ok; ++pre) {
        madvance();
        if (!mend) ok = gen_mask();
      }
    }
    int gs = 0;
    for (int k = 0; ok && k * G < total_units; ++k) {
      const int u = unit_at(k);
      if (u >= total_units) continue;
      const Unit U = decode(u);
      for (int i = 0; i < U.nsteps && ok; ++i) {
        const int gi = gs + i;
        if (C::HAS_DQ) {
          const int x = set_of(gi);
          ok = warp_wait_all(bar(B_DQFULL + x), set_phase(gi), wc);
          if (!ok) break;
          tc_fence_after();
          const int h = step_head(U, i), q0 = step_qblk(U, i) * C::BM;
          const int nvalid = min(C::BM, p.Nq - q0);
          float *acc = p.dq_acc + (((size_t)(U.b * p.Hq + h)) * p.Nq + q0) * C::D + t;
          const uint32_t src = tmem + lane_off + C::TM_SET0 + x * C::SET_STRIDE + C::TM_DQ;
          // chunks 0 and 1 (the elementwise warpgroups take chunks 2 and 3)
          uint32_t v0[32], v1[32];
          tmem_ld32(src, v0);
          tmem_ld32(src + 32, v1);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(bar(B_DQEMPTY + x));
          reduce_dq_chunk<C>(v0, acc, 0, t, nvalid);
          reduce_dq_chunk<C>(v1, acc, 1, t, nvalid);
        }
        if (DROP) {
          madvance();
          if (!mend) ok = gen_mask();
        }
      }
      gs += U.nsteps;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_ALLOC);
  }
}

// ---------------------------------------------------------------------------
// dkdv for d <= 128 with 128-row query blocks.
//
// An M = 128 tcgen05 MMA costs about as much for N = 64 as for N = 128, so
// S^T, dP^T and dQ^T are computed for 128 query columns at a time.  TMEM then
// holds dV, dK and one set of scores:
//     d = 128: dV [0,128) dK [128,256) A [256,384) B [384,512)
//     d =  64: dV [0, 64) dK [ 64,128) A [128,256) B [256,384)
// A receives S^T(i), which the elementwise stage overwrites in place with
// bf16 P^T and dS^T; B receives dP^T(i) and then dQ^T(i).  The elementwise
// stage runs in two phases so the tensor cores are not left idle while it
// works:
//     phase 1 (needs S^T):  P^T = exp2(S^T * scale*log2e - L2)  -> dV(i) may start
//     phase 2 (needs dP^T): dS^T = P^T * (dP^T - D)            -> dK(i), dQ^T(i)
// MMA issue order per step:  dV(i)  dK(i)  S^T(i+1)  dQ^T(i)  dP^T(i+1).
// S^T(i+1) only replaces what dV(i) and dK(i), issued before it, read;
// dP^T(i+1) waits until the readout warps hold dQ^T(i) in registers.  Phase 1
// of step i+1 then overlaps dQ^T(i), its readout and dP^T(i+1), and phase 2
// overlaps dV(i+1).  P^T is kept in registers between the phases in bf16, the
// precision the dV MMA also uses.
//
// Two step orders (BwdWideCfg::EARLY_S):
//   default  dV(i)  dK(i)  S^T(i+1)  dQ^T(i)  dP^T(i+1), dK's A operand (dS^T)
//            from TMEM: S^T(i+1) waits for phase 2 of step i;
//   EARLY_S  dV(i)  S^T(i+1)  dQ^T(i)  dK(i)  dP^T(i+1), dS^T only in shared
//            memory (A operand of dK, K-major): S^T(i+1) is computed while
//            phase 2 of step i runs, so phase 1 of step i+1 follows phase 2 at
//            once.  Measured on B200 (dK/dV kernel, same build otherwise):
//            d = 64 faster (causal B8 H16 N2048: 0.745 -> 0.684 ms), d = 128
//            slower (causal B4 H16 N4096: 0.875 -> 0.952 ms): the extra shared-
//            memory operand reads and the dQ reductions that then overlap the
//            tensor-core work cost more than the shorter chain gains.
// With EARLY_S, phase 2 writes dS^T(i) to shared memory only after dP^T(i)
// has completed, which implies dQ^T(i-1) and dK(i-1), issued before it, are
// done reading the previous dS^T.
//
// Persistent CTAs, one per SM.  CTA c starts with unit c of the list; the
// producer takes the next unit from a counter in the workspace (atomicAdd;
// the prep stage zeroes it) once it has issued all loads of its current unit,
// so the SM that frees up first gets the heaviest unit left, and it hands the
// unit to the other roles through a four-entry shared-memory queue.  The next
// unit's K and V are prefetched into L2 at that point and loaded into shared
// memory when the current unit's last MMA completes; its first Q/dO tiles are
// already in the ring.  The epilogue reads dV and dK out of TMEM and releases
// them (acc_empty) before storing, and the next unit's first dV/dK MMAs wait
// for that release.  Units are listed in groups of key/value heads whose
// f32 dQ accumulator, Q and dO take about 32 MB (the dQ reductions of a group
// stay in L2), the key blocks with most query blocks first within a group
// (causal).  Measured on B200 against one CTA per unit with the same steps:
// causal B4 H16 N4096 d128 0.889 -> 0.854 ms, GQA B1 Hq32 Hkv8 N16384
// 6.35 -> 6.12 ms, causal B64 H16 N512 d128 0.520 -> 0.453 ms.
//
// Warps: 0-7 elementwise (two warpgroups, 64 query columns each; warpgroup 0
// writes dV and warpgroup 1 dK at the end of a unit), 8-15 dQ^T readout (two
// warps per TMEM lane quarter, two 32-column chunks each, float32 reductions
// into the accumulator), 16 TMA producer, 17 MMA issuer (both in lane 0).
// EARLY_S_: the step order that issues S^T(i+1) right after dV(i) and takes
// dK's A operand (dS^T) from shared memory (see the comment block above).
// MASKGEN_ (the dropout instances): the readout warps, which wait most of a
// step, evaluate the Philox words of the dropout mask two steps ahead into a
// double-buffered bit array in shared memory (one bit per key row and query
// column, 2 KB a step), so the elementwise stage reads 64 bits instead of
// evaluating 16 Philox calls per step on the critical path.
template <int D_, int QS_, bool EARLY_S_, bool MASKGEN_ = false>
struct BwdWideCfg {
  static constexpr int D = D_, QS = QS_;
  static constexpr bool EARLY_S = EARLY_S_;
  static constexpr bool MASKGEN = MASKGEN_;
  static constexpr int BN = 128, BM = 128;
  static constexpr int DCH = D / 64;
  static constexpr int KV_CHUNK = BN * 128;
  static constexpr int KV_TILE = KV_CHUNK * DCH;
  static constexpr int Q_CHUNK = BM * 128;
  static constexpr int Q_TILE = Q_CHUNK * DCH;
  static constexpr int DS_CHUNK = BN * 128;        // 64 query columns of dS^T (bf16)
  static constexpr int DS_TILE = DS_CHUNK * 2;
  static constexpr int ROWVEC = BM * 4;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_TILE;    // must directly follow K (d = 64 dQ MMA)
  static constexpr int OFF_Q = OFF_V + KV_TILE;
  static constexpr int OFF_DO = OFF_Q + QS * Q_TILE;
  static constexpr int OFF_DS = OFF_DO + QS * Q_TILE;
  static constexpr int OFF_L2 = OFF_DS + DS_TILE;
  static constexpr int OFF_DD = OFF_L2 + QS * ROWVEC;
  static constexpr int OFF_MASK = OFF_DD + QS * ROWVEC;   // [2][128 key rows][128 query bits]
  static constexpr int MASK_BUF = BN * BM / 8;
  static constexpr int OFF_BAR = OFF_MASK + (MASKGEN ? 2 * MASK_BUF : 0);
  // kv, kc, q_full[QS], q_empty[QS], s_full, dp_full, p_full, ds_full,
  // dq_full, dq_empty, final, drain, acc_empty, unit_full[4], unit_empty[4],
  // mask_full[2], mask_empty[2]
  static constexpr int NBAR = 2 + 2 * QS + 9 + 8 + 4;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;   // tmem slot, abort flag, unit queue[4]
  static constexpr int SMEM = OFF_MISC + 32;
  static constexpr int TM_DV = 0, TM_DK = D, TM_A = 2 * D, TM_B = 2 * D + 128;
  static constexpr int TM_ALLOC = 512;
  static constexpr int THREADS = 18 * 32;
  static constexpr int READOUT_WARP0 = 8, PRODUCER_WARP = 16, MMA_WARP = 17;
  static_assert(TM_B + 128 <= TM_ALLOC, "TMEM");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(D == 64 || D == 128, "wide path is for d = 64 and 128");
};

template <class C, bool DROP>
__global__ void __launch_bounds__(C::THREADS, 1)
    bwd_wide_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const BwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The 128-byte swizzled tiles need a 1024-byte aligned base.
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(p.err, kErrConfig);
    return;
  }
  uint8_t *smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  uint64_t *bars = (uint64_t *)(smem + C::OFF_BAR);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const int B_KV = 0, B_KC = 1, B_QFULL = 2, B_QEMPTY = 2 + C::QS, B_SFULL = 2 + 2 * C::QS,
            B_DPFULL = B_SFULL + 1, B_PFULL = B_SFULL + 2, B_DSFULL = B_SFULL + 3,
            B_DQFULL = B_SFULL + 4, B_DQEMPTY = B_SFULL + 5, B_FINAL = B_SFULL + 6,
            B_DRAIN = B_SFULL + 7, B_ACCEMPTY = B_SFULL + 8, B_UFULL = B_SFULL + 9,
            B_UEMPTY = B_UFULL + 4, B_MFULL = B_UEMPTY + 4, B_MEMPTY = B_MFULL + 2;
  static_assert(DROP == C::MASKGEN, "dropout instances take their mask from the readout warps");
  uint32_t *tmem_slot = (uint32_t *)(smem + C::OFF_MISC);
  volatile int *abort_flag = (volatile int *)(smem + C::OFF_MISC + 4);
  volatile int *s_queue = (volatile int *)(smem + C::OFF_MISC + 16);   // unit of the k-th turn, k % 4
  const float *s_l2 = (const float *)(smem + C::OFF_L2);
  const float *s_dd = (const float *)(smem + C::OFF_DD);

  const int warp = warp_id_uniform();
  const int lane = threadIdx.x & 31;
  const int g = p.Hq / p.Hkv;

  // Work units: (batch, key/value head, 128-row key block).  The unit list
  // runs over groups of hg heads one after the other; inside a group the
  // key blocks with the most query blocks come first (causal), heads
  // interleaved.  Persistent CTAs (one per SM): CTA c starts with unit c;
  // after that the producer takes the next unit of the list from a counter
  // in the workspace (atomicAdd) when it has issued the loads of its current
  // one, so the SM that frees up first gets the heaviest unit left (the order
  // a hardware block scheduler would give, without a CTA's set-up and
  // teardown between units).  The producer hands each unit to the other
  // roles through a four-entry queue in shared memory (-1 ends the
  // sequence); barrier phases follow the count of units (uc) and of steps
  // (gs) this CTA has processed.
  const int total_units = p.nkb * p.BHkv;
  const int G = (int)gridDim.x;
  struct Unit {
    int bhkv, b, hkv, kv0, i0, nq_eff, nsteps;
  };
  auto decode = [&](int u) {
    Unit U;
    const int grp = u / (p.hg * p.nkb), wu = u % (p.hg * p.nkb);
    const int hn = min(p.hg, p.BHkv - grp * p.hg);
    const int jblk = wu / hn;
    U.bhkv = grp * p.hg + wu % hn;
    U.b = U.bhkv / p.Hkv;
    U.hkv = U.bhkv % p.Hkv;
    U.kv0 = jblk * C::BN;
    U.i0 = p.causal ? U.kv0 / C::BM : 0;   // first query block that sees this key block
    U.nq_eff = p.nqb - U.i0;
    U.nsteps = U.nq_eff > 0 ? g * U.nq_eff : 0;
    return U;
  };
  auto step_head = [&](const Unit &U, int s) { return U.hkv * g + s / U.nq_eff; };
  auto step_qblk = [&](const Unit &U, int s) { return U.i0 + s % U.nq_eff; };

  if (threadIdx.x == 0) {
    mbar_init(bar(B_KV), 1);
    mbar_init(bar(B_KC), 256);
    for (int s = 0; s < C::QS; ++s) {
      mbar_init(bar(B_QFULL + s), 1);
      mbar_init(bar(B_QEMPTY + s), 1);
    }
    mbar_init(bar(B_SFULL), 1);
    mbar_init(bar(B_DPFULL), 1);
    mbar_init(bar(B_PFULL), 256);
    mbar_init(bar(B_DSFULL), 256);
    mbar_init(bar(B_DQFULL), 1);
    mbar_init(bar(B_DQEMPTY), 256);
    mbar_init(bar(B_FINAL), 1);
    mbar_init(bar(B_DRAIN), 1);
    mbar_init(bar(B_ACCEMPTY), 256);
    for (int s = 0; s < 4; ++s) {
      mbar_init(bar(B_UFULL + s), 1);
      mbar_init(bar(B_UEMPTY + s), 17);   // MMA issuer + 8 elementwise + 8 readout warps
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_MFULL + s), 256);    // the readout threads wrote their mask bits
      mbar_init(bar(B_MEMPTY + s), 256);   // the elementwise threads read theirs
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), C::TM_ALLOC);
    tmem_relinquish();
  }
  if (warp == C::PRODUCER_WARP && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmDO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  WaitCtx wc{p.err, abort_flag, kWaitLimitNs};

  if (warp == C::PRODUCER_WARP) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int last_phase[C::QS];
      for (int s = 0; s < C::QS; ++s) last_phase[s] = -1;
      int kv_phase = -1;
      bool ok = true;
      int uc = 0, gs = 0;
      // Q_i, dO_i and the row slices of L2 and D of step i of unit U
      auto load_step = [&](const Unit &U, int i) {
        const int gi = gs + i;
        const int st = gi % C::QS;
        const uint32_t ph = (gi / C::QS) & 1;
        if (!bounded_wait(bar(B_QEMPTY + st), ph ^ 1, wc)) return false;
        const int h = step_head(U, i), qb = step_qblk(U, i);
        const int bh = U.b * p.Hq + h;
        const size_t vrow = (size_t)bh * p.npad + (size_t)qb * C::BM;
        const uint32_t fb = bar(B_QFULL + st);
        mbar_arrive_expect_tx(fb, 2 * C::Q_TILE + 2 * C::ROWVEC);
        for (int c = 0; c < C::DCH; ++c) {
          tma_load_3d(sbase + C::OFF_Q + st * C::Q_TILE + c * C::Q_CHUNK, &tmQ, fb, c * 64,
                      qb * C::BM, bh);
          tma_load_3d(sbase + C::OFF_DO + st * C::Q_TILE + c * C::Q_CHUNK, &tmDO, fb, c * 64,
                      qb * C::BM, bh);
        }
        bulk_load(sbase + C::OFF_L2 + st * C::ROWVEC, p.l2 + vrow, C::ROWVEC, fb);
        bulk_load(sbase + C::OFF_DD + st * C::ROWVEC, p.dsum + vrow, C::ROWVEC, fb);
        last_phase[st] = ph;
        return true;
      };
      int u = (int)blockIdx.x;
      for (int k = 0; ok; ++k) {
        // publish this turn's unit (or the end of the sequence)
        ok = bounded_wait(bar(B_UEMPTY + (k & 3)), ((k >> 2) & 1) ^ 1, wc);
        if (!ok) break;
        s_queue[k & 3] = u < total_units ? u : -1;
        mbar_arrive(bar(B_UFULL + (k & 3)));
        if (u >= total_units) break;
        const Unit U = decode(u);
        if (U.nsteps == 0) {
          u = G + atomicAdd(p.sched, 1);
          continue;
        }
        // the first ring slots of this unit, then K and V once the previous
        // unit's MMAs (the last readers of K and V) are done, then the rest
        const int pre = min(C::QS, U.nsteps);
        for (int i = 0; i < pre && ok; ++i) ok = load_step(U, i);
        if (ok && uc > 0) ok = bounded_wait(bar(B_FINAL), (uc - 1) & 1, wc);
        if (!ok) break;
        mbar_arrive_expect_tx(bar(B_KV), 2 * C::KV_TILE);
        for (int c = 0; c < C::DCH; ++c) {
          tma_load_3d(sbase + C::OFF_K + c * C::KV_CHUNK, &tmK, bar(B_KV), c * 64, U.kv0, U.bhkv);
          tma_load_3d(sbase + C::OFF_V + c * C::KV_CHUNK, &tmV, bar(B_KV), c * 64, U.kv0, U.bhkv);
        }
        kv_phase = uc & 1;
        for (int i = pre; i < U.nsteps && ok; ++i) ok = load_step(U, i);
        gs += U.nsteps;
        ++uc;
        // the next unit, taken once this one's loads are all issued; its K
        // and V tiles go to L2 now, so their load after this unit's last MMA
        // does not wait on DRAM
        u = G + atomicAdd(p.sched, 1);
        if (u < total_units) {
          const Unit N = decode(u);
          for (int c = 0; c < C::DCH; ++c) {
            tma_prefetch_l2_3d(&tmK, c * 64, N.kv0, N.bhkv);
            tma_prefetch_l2_3d(&tmV, c * 64, N.kv0, N.bhkv);
          }
        }
      }
      if (!ok) {
        if (kv_phase >= 0) (void)drain_wait(bar(B_KV), kv_phase, p.err, kWaitLimitNs);
        for (int s = 0; s < C::QS; ++s)
          if (last_phase[s] >= 0) (void)drain_wait(bar(B_QFULL + s), last_phase[s], p.err, kWaitLimitNs);
      }
    }
    __syncwarp();
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t IDESC_SP = idesc_bf16(128, C::BM, 0, 0);  // S^T, dP^T
    constexpr uint32_t IDESC_KV = idesc_bf16(128, C::D, 0, 1);   // dV, dK: A TMEM, B MN-major
    constexpr uint32_t IDESC_DQ = idesc_bf16(128, C::BM, 1, 1);  // dQ^T: both MN-major
    const uint64_t dK_km = sw128_desc(sbase + C::OFF_K, 16, 1024);
    const uint64_t dV_km = sw128_desc(sbase + C::OFF_V, 16, 1024);
    const uint64_t dK_mn = sw128_desc(sbase + C::OFF_K, C::KV_CHUNK, 1024);
    const uint64_t dQ_km = sw128_desc(sbase + C::OFF_Q, 16, 1024);
    const uint64_t dQ_mn = sw128_desc(sbase + C::OFF_Q, C::Q_CHUNK, 1024);
    const uint64_t dO_km = sw128_desc(sbase + C::OFF_DO, 16, 1024);
    const uint64_t dO_mn = sw128_desc(sbase + C::OFF_DO, C::Q_CHUNK, 1024);
    const uint64_t dS_mn = sw128_desc(sbase + C::OFF_DS, C::DS_CHUNK, 1024);
    const uint64_t dS_km = sw128_desc(sbase + C::OFF_DS, 16, 1024);
    // S^T = (K-c) Q^T (A region), dP^T = V dO^T (B region); K = d, 16 per MMA
    auto issue_SP = [&](uint64_t a0, uint64_t b0, int st, uint32_t dst) {
      const uint64_t bt = desc_add(b0, st * C::Q_TILE);
#pragma unroll
      for (int kk = 0; kk < C::D / 16; ++kk) {
        const uint32_t okv = (kk >> 2) * C::KV_CHUNK + (kk & 3) * 32;
        const uint32_t oq = (kk >> 2) * C::Q_CHUNK + (kk & 3) * 32;
        mma_ss(dst, desc_add(a0, okv), desc_add(bt, oq), IDESC_SP, kk > 0);
      }
    };
    // dV += P^T dO_i, dK += dS^T Q_i: K = 128 query rows, 16 per MMA; query
    // rows 16 kk .. 16 kk + 15 sit in the 32-column block kk / 2 of A: P^T at
    // 32 (kk / 2) + 8 (kk % 2), dS^T 16 columns further.
    auto issue_grad = [&](uint64_t b0, int st, uint32_t acc, int col, bool first) {
      const uint64_t bt = desc_add(b0, st * C::Q_TILE);
#pragma unroll
      for (int kk = 0; kk < C::BM / 16; ++kk)
        mma_ts(tmem + acc, tmem + C::TM_A + (kk >> 1) * 32 + (kk & 1) * 8 + col,
               desc_add(bt, kk * 2048), IDESC_KV, (!first) || kk > 0);
    };
    // EARLY_S: dK += dS^T Q_i with dS^T read from shared memory (K-major: key
    // rows of 64-query-column chunks), so A is free for S^T(i+1) once dV(i)
    // has read P^T(i).
    auto issue_dk_smem = [&](int st, bool first) {
      const uint64_t bt = desc_add(dQ_mn, st * C::Q_TILE);
#pragma unroll
      for (int kk = 0; kk < C::BM / 16; ++kk)
        mma_ss(tmem + C::TM_DK, desc_add(dS_km, (kk >> 2) * C::DS_CHUNK + (kk & 3) * 32),
               desc_add(bt, kk * 2048), IDESC_KV, (!first) || kk > 0);
    };
    // dQ^T = A^T dS^T, K = 128 key rows (16 per MMA), M = 128 rows of A^T:
    // (K-c)^T for d = 128, [(K-c)^T ; V^T] for d = 64 (the V half unused).
    auto issue_dq = [&]() {
#pragma unroll
      for (int kk = 0; kk < C::BN / 16; ++kk)
        mma_ss(tmem + C::TM_B, desc_add(dK_mn, kk * 2048), desc_add(dS_mn, kk * 2048), IDESC_DQ,
               kk > 0);
    };
    if (lane == 0) {
      bool ok = true;
      int uc = 0, gs = 0;
      for (int k = 0; ok; ++k) {
        ok = bounded_wait(bar(B_UFULL + (k & 3)), (k >> 2) & 1, wc);
        if (!ok) break;
        const int u = s_queue[k & 3];
        mbar_arrive(bar(B_UEMPTY + (k & 3)));
        if (u < 0) break;
        const Unit U = decode(u);
        const int nsteps = U.nsteps;
        if (nsteps == 0) continue;
        // this unit's K - c in place, Q_0 loaded
        ok = bounded_wait(bar(B_KC), uc & 1, wc);
        if (ok) ok = bounded_wait(bar(B_QFULL + gs % C::QS), (gs / C::QS) & 1, wc);
        if (!ok) break;
        tc_fence_after();
        issue_SP(dK_km, dQ_km, gs % C::QS, tmem + C::TM_A);
        mma_commit(bar(B_SFULL));
        // B: the previous unit's last dQ^T has been read out
        if (gs > 0) {
          ok = bounded_wait(bar(B_DQEMPTY), (gs - 1) & 1, wc);
          if (!ok) break;
          tc_fence_after();
        }
        issue_SP(dV_km, dO_km, gs % C::QS, tmem + C::TM_B);
        mma_commit(bar(B_DPFULL));
        for (int i = 0; i < nsteps && ok; ++i) {
          const int gi = gs + i;
          const int st = gi % C::QS;
          const uint32_t par = gi & 1;
          const int st1 = (gi + 1) % C::QS;
          const uint32_t ph1 = ((gi + 1) / C::QS) & 1;
          ok = bounded_wait(bar(B_PFULL), par, wc);
          // dV(0) and dK(0) start the accumulators afresh: the previous
          // unit's epilogue must have read them out of TMEM
          if (ok && i == 0 && uc > 0) ok = bounded_wait(bar(B_ACCEMPTY), (uc - 1) & 1, wc);
          if (!ok) break;
          tc_fence_after();
          issue_grad(dO_mn, st, C::TM_DV, 0, i == 0);
          if constexpr (C::EARLY_S) {
            // dV(i)  S^T(i+1)  dQ^T(i)  dK(i)  dP^T(i+1)
            if (i + 1 < nsteps) {
              // S^T(i+1) over A: phase 1 has read S^T(i) and dV(i), issued
              // before it, is the last reader of P^T(i)
              ok = bounded_wait(bar(B_QFULL + st1), ph1, wc);
              if (!ok) break;
              tc_fence_after();
              issue_SP(dK_km, dQ_km, st1, tmem + C::TM_A);
              mma_commit(bar(B_SFULL));
            }
            // phase 2 has read dP^T(i) out of B and put dS^T(i) in shared memory
            ok = bounded_wait(bar(B_DSFULL), par, wc);
            if (!ok) break;
            tc_fence_after();
            issue_dq();
            mma_commit(bar(B_DQFULL));
            issue_dk_smem(st, i == 0);
            mma_commit(bar(B_QEMPTY + st));
          } else {
            // dV(i)  dK(i)  S^T(i+1)  dQ^T(i)  dP^T(i+1)
            ok = bounded_wait(bar(B_DSFULL), par, wc);
            if (!ok) break;
            tc_fence_after();
            issue_grad(dQ_mn, st, C::TM_DK, 16, i == 0);
            mma_commit(bar(B_QEMPTY + st));
            if (i + 1 < nsteps) {
              ok = bounded_wait(bar(B_QFULL + st1), ph1, wc);
              if (!ok) break;
              tc_fence_after();
              issue_SP(dK_km, dQ_km, st1, tmem + C::TM_A);
              mma_commit(bar(B_SFULL));
            }
            issue_dq();
            mma_commit(bar(B_DQFULL));
          }
          if (i + 1 < nsteps) {
            ok = bounded_wait(bar(B_DQEMPTY), par, wc);
            if (!ok) break;
            tc_fence_after();
            issue_SP(dV_km, dO_km, st1, tmem + C::TM_B);
            mma_commit(bar(B_DPFULL));
          }
        }
        if (!ok) break;
        // the unit's accumulators are final once its MMAs complete; this also
        // releases K and V to the producer
        mma_commit(bar(B_FINAL));
        gs += nsteps;
        ++uc;
      }
      if (!ok) {
        mma_commit(bar(B_DRAIN));
        (void)drain_wait(bar(B_DRAIN), 0, p.err, kWaitLimitNs);
      }
    }
    __syncwarp();
  } else if (warp < C::READOUT_WARP0) {
    // ------------------------------------------------ elementwise stage
    const int wg = warp >> 2;                      // query columns [64 wg, 64 wg + 64)
    const int r = threadIdx.x & 127;               // key row within the block = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tA = tmem + lane_off + C::TM_A;
    const uint32_t tB = tmem + lane_off + C::TM_B;
    bool ok = true;
    int uc = 0, gs = 0;
    for (int k = 0; ok; ++k) {
      ok = warp_wait_all(bar(B_UFULL + (k & 3)), (k >> 2) & 1, wc);
      if (!ok) break;
      const int u = s_queue[k & 3];
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_UEMPTY + (k & 3)));
      if (u < 0) break;
      const Unit U = decode(u);
      const int nsteps = U.nsteps;
      const int kv = U.kv0 + r;
      const bool kv_live = kv < p.Nk;
      if (nsteps == 0) {
        // no query row sees this key block: its gradients are zero
        if (kv_live) {
          __nv_bfloat16 *dst = (wg ? p.dk : p.dv) + ((size_t)U.bhkv * p.Nk + kv) * C::D;
          for (int e = 0; e < C::D / 8; ++e) reinterpret_cast<uint4 *>(dst)[e] = make_uint4(0, 0, 0, 0);
        }
        continue;
      }
      {
        // K row r -> K - c in place (same swizzled layout; rows past Nk were
        // zero-filled and stay zero).  Warpgroup wg takes the 16-byte units
        // 4 wg .. 4 wg + 3 of each 128-byte chunk of the row; the entries of
        // c they need are read before K has arrived.
        const float *cv = p.cvec + (size_t)U.bhkv * C::D;
        float cc[C::DCH][32];
#pragma unroll
        for (int ch = 0; ch < C::DCH; ++ch)
#pragma unroll
          for (int e4 = 0; e4 < 4; ++e4) {
            const int col = ch * 64 + (((4 * wg + e4) ^ (r & 7)) << 3);
            const float4 c_lo = *reinterpret_cast<const float4 *>(cv + col);
            const float4 c_hi = *reinterpret_cast<const float4 *>(cv + col + 4);
            cc[ch][8 * e4 + 0] = c_lo.x; cc[ch][8 * e4 + 1] = c_lo.y;
            cc[ch][8 * e4 + 2] = c_lo.z; cc[ch][8 * e4 + 3] = c_lo.w;
            cc[ch][8 * e4 + 4] = c_hi.x; cc[ch][8 * e4 + 5] = c_hi.y;
            cc[ch][8 * e4 + 6] = c_hi.z; cc[ch][8 * e4 + 7] = c_hi.w;
          }
        ok = warp_wait_all(bar(B_KV), uc & 1, wc);
        if (!ok) break;
#pragma unroll
        for (int ch = 0; ch < C::DCH; ++ch) {
          uint8_t *row = smem + C::OFF_K + ch * C::KV_CHUNK + r * 128;
#pragma unroll
          for (int e4 = 0; e4 < 4; ++e4) {
            const int e8 = 4 * wg + e4;
            uint4 v = *reinterpret_cast<const uint4 *>(row + (e8 << 4));
            uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 h2 = *reinterpret_cast<__nv_bfloat162 *>(&w[e]);
              const float2 f = __bfloat1622float2(h2);
              w[e] = kv_live ? pack_bf16x2(f.x - cc[ch][8 * e4 + 2 * e], f.y - cc[ch][8 * e4 + 2 * e + 1])
                             : 0u;
            }
            *reinterpret_cast<uint4 *>(row + (e8 << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(bar(B_KC));
      }
      for (int i = 0; i < nsteps && ok; ++i) {
        const int gi = gs + i;
        const int st = gi % C::QS;
        const uint32_t par = gi & 1;
        const int q0 = step_qblk(U, i) * C::BM;
        ok = warp_wait_all(bar(B_QFULL + st), (gi / C::QS) & 1, wc);
        if (ok) ok = warp_wait_all(bar(B_SFULL), par, wc);
        if (!ok) break;
        tc_fence_after();
        // ---- phase 1: P^T for query columns [64 wg, 64 wg + 64), 16 at a time
        uint32_t pkeep[4][8];
        uint32_t keepbits[2] = {0u, 0u};               // dropout: bit c = column 64 wg + c kept
        if (DROP) {
          ok = warp_wait_all(bar(B_MFULL + (gi & 1)), (gi >> 1) & 1, wc);
          if (!ok) break;
          const uint2 kb = *reinterpret_cast<const uint2 *>(smem + C::OFF_MASK + (gi & 1) * C::MASK_BUF +
                                                            r * (C::BM / 8) + 8 * wg);
          keepbits[0] = kb.x;
          keepbits[1] = kb.y;
          mbar_arrive(bar(B_MEMPTY + (gi & 1)));
        }
#pragma unroll
        for (int sb = 0; sb < 4; ++sb) {
          const int c0 = 64 * wg + 16 * sb;
          uint32_t sv[16];
          tmem_ld16(tA + c0, sv);
          tmem_wait_ld();
          const float4 *l4 = reinterpret_cast<const float4 *>(s_l2 + st * C::BM + c0);
          // causal: key kv is hidden from query q when kv > q; key rows past
          // Nk (zero-filled) are masked so they add nothing anywhere.  Query
          // rows past Nq have L2 = +inf, so their P is 0.
          const int first_vis = !kv_live ? 16 : (p.causal ? kv - (q0 + c0) : 0);
          float pr[16];
#pragma unroll
          for (int e4 = 0; e4 < 4; ++e4) {
            const float4 lq = l4[e4];
            const float lv[4] = {lq.x, lq.y, lq.z, lq.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = 4 * e4 + e;
              const float pv = fast_exp2(fmaf(__uint_as_float(sv[c]), p.scale_log2, -lv[e]));
              pr[c] = (c >= first_vis) ? pv : 0.f;
            }
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) pkeep[sb][e] = pack_bf16x2(pr[2 * e], pr[2 * e + 1]);
          // P^T of query columns 32h + 16(sb%2) + [0,16) -> A columns 32h + 8(sb%2) + [0,8),
          // all of which this thread has already read.  With dropout the dV
          // operand is P^T * Z; pkeep keeps P^T for dS.
          if (DROP) {
            const uint32_t m16 = (keepbits[sb >> 1] >> (16 * (sb & 1))) & 0xffffu;
            uint32_t pm[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              pm[e] = pack_bf16x2(((m16 >> (2 * e)) & 1u) ? pr[2 * e] : 0.f,
                                  ((m16 >> (2 * e + 1)) & 1u) ? pr[2 * e + 1] : 0.f);
            tmem_st8(tA + 32 * (2 * wg + (sb >> 1)) + 8 * (sb & 1), pm);
          } else {
            tmem_st8(tA + 32 * (2 * wg + (sb >> 1)) + 8 * (sb & 1), pkeep[sb]);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_PFULL));
        // ---- phase 2: dS^T = P^T (dP^T - D)
        ok = warp_wait_all(bar(B_DPFULL), par, wc);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int sb = 0; sb < 4; ++sb) {
          const int c0 = 64 * wg + 16 * sb;
          uint32_t dv[16];
          tmem_ld16(tB + c0, dv);
          tmem_wait_ld();
          const float4 *d4 = reinterpret_cast<const float4 *>(s_dd + st * C::BM + c0);
          uint32_t dk[8];
#pragma unroll
          for (int e4 = 0; e4 < 4; ++e4) {
            const float4 dq4 = d4[e4];
            const float dd[4] = {dq4.x, dq4.y, dq4.z, dq4.w};
            float ds[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = 4 * e4 + e;
              const uint32_t pp = pkeep[sb][c >> 1];
              const float pv = __uint_as_float((c & 1) ? (pp & 0xffff0000u) : (pp << 16));
              float dpv = __uint_as_float(dv[c]);
              if (DROP) dpv = ((keepbits[sb >> 1] >> (16 * (sb & 1) + c)) & 1u) ? dpv * p.drop_scale : 0.f;
              ds[e] = pv * (dpv - dd[e]);
            }
            dk[2 * e4] = pack_bf16x2(ds[0], ds[1]);
            dk[2 * e4 + 1] = pack_bf16x2(ds[2], ds[3]);
          }
          // dS^T -> A (the dK operand) unless EARLY_S, where S^T(i+1) may
          // already be there and dK reads dS^T from shared memory
          if constexpr (!C::EARLY_S) tmem_st8(tA + 32 * (2 * wg + (sb >> 1)) + 16 + 8 * (sb & 1), dk);
          // dS^T row r -> shared memory (B operand of the dQ^T MMA, and with
          // EARLY_S the A operand of dK: 64-column chunks of 128-byte swizzled
          // rows; 16-byte unit u of row r sits at unit u ^ (r % 8))
          uint8_t *dsrow = smem + C::OFF_DS + (c0 >> 6) * C::DS_CHUNK + r * 128;
          const int u0 = (c0 & 63) >> 3;
#pragma unroll
          for (int c = 0; c < 2; ++c)
            *reinterpret_cast<uint4 *>(dsrow + (((u0 + c) ^ (r & 7)) << 4)) =
                make_uint4(dk[4 * c], dk[4 * c + 1], dk[4 * c + 2], dk[4 * c + 3]);
        }
        fence_proxy_async_smem();
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_DSFULL));
      }
      if (!ok) break;
      // ---------------------------------------------------- epilogue
      // warpgroup 0 writes dV, warpgroup 1 writes dK (one key row per thread);
      // the accumulators are released once read, before the stores complete
      ok = warp_wait_all(bar(B_FINAL), uc & 1, wc);
      if (!ok) break;
      tc_fence_after();
      {
        const size_t rowoff = ((size_t)U.bhkv * p.Nk + (kv_live ? kv : 0)) * C::D;
        const uint32_t src = tmem + lane_off + (wg ? C::TM_DK : C::TM_DV);
        __nv_bfloat16 *dst = (wg ? p.dk : p.dv) + rowoff;
        const float mul = wg ? p.scale : (DROP ? p.drop_scale : 1.f);
#pragma unroll 1
        for (int c = 0; c < C::D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(src + c * 32, v);
          tmem_wait_ld();
          if (c == C::D / 32 - 1) {
            tc_fence_before();
            mbar_arrive(bar(B_ACCEMPTY));
          }
          uint32_t pkd[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pkd[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * mul, __uint_as_float(v[2 * e + 1]) * mul);
          if (kv_live) {
            uint4 *o = reinterpret_cast<uint4 *>(dst + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) o[e] = make_uint4(pkd[4 * e], pkd[4 * e + 1], pkd[4 * e + 2], pkd[4 * e + 3]);
          }
        }
      }
      gs += nsteps;
      ++uc;
    }
  } else if (warp < C::PRODUCER_WARP) {
    // ------------------------------------------------ dQ^T readout
    const int quad = warp & 3;
    const int t = quad * 32 + lane;                  // TMEM lane = row d of dQ^T
    const int ch0 = ((warp - C::READOUT_WARP0) >> 2) * 2;   // chunks ch0, ch0 + 1
    const uint32_t src = tmem + ((uint32_t)(quad * 32) << 16) + C::TM_B + ch0 * 32;
    const bool live_rows = quad * 32 < C::D;    // d = 64: lanes 64..127 carry no dQ
    bool ok = true;
    // Units of the sequence by turn, fetched from the queue by whichever
    // cursor reaches a turn first (the mask cursor runs at most two steps
    // ahead of the readout cursor, so eight entries are plenty).
    int ucache[8];
    int fetched = 0;
    auto unit_of = [&](int k, int &u) {
      while (fetched <= k) {
        if (!warp_wait_all(bar(B_UFULL + (fetched & 3)), (fetched >> 2) & 1, wc)) return false;
        ucache[fetched & 7] = s_queue[fetched & 3];
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_UEMPTY + (fetched & 3)));
        ++fetched;
      }
      u = ucache[k & 7];
      return true;
    };
    // A cursor over the steps of the sequence: turn k, its unit U, step i of
    // the unit and g, the running step count (the elementwise stage's gs + i).
    struct Cursor {
      int k, i, g;
      bool end;
      Unit U;
    };
    auto advance = [&](Cursor &c) {
      if (c.end) return true;
      if (c.k >= 0 && c.i + 1 < c.U.nsteps) {
        ++c.i;
        ++c.g;
        return true;
      }
      for (;;) {
        int u;
        if (!unit_of(c.k + 1, u)) return false;
        ++c.k;
        if (u < 0) {
          c.end = true;
          return true;
        }
        c.U = decode(u);
        if (c.U.nsteps > 0) {
          c.i = 0;
          ++c.g;
          return true;
        }
      }
    };
    // Dropout keep bits of step c.g: thread tt evaluates the Philox counters
    // of key rows 4 kq .. 4 kq + 3 (counter word 0 = key / 4, word j of the
    // result = key row 4 kq + j) for query columns 16 qg .. 16 qg + 15 of the
    // step, the counters the forward used, and stores 16 bits per key row.
    auto gen_mask = [&](const Cursor &c) {
      const int buf = c.g & 1;
      if (!warp_wait_all(bar(B_MEMPTY + buf), ((c.g >> 1) & 1) ^ 1, wc)) return false;
      const int tt = (warp - C::READOUT_WARP0) * 32 + lane;
      const int kq = tt >> 3, qg = tt & 7;
      const uint32_t kc = (uint32_t)((c.U.kv0 >> 2) + kq);
      const uint32_t q = (uint32_t)(step_qblk(c.U, c.i) * C::BM + 16 * qg);
      const uint32_t bhq = (uint32_t)(c.U.b * p.Hq + step_head(c.U, c.i));
      uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
#pragma unroll 4
      for (int e = 0; e < 16; ++e) {
        const uint4 R = philox4x32_10(kc, q + e, bhq, p.drop_off, p.seed_lo, p.seed_hi);
        m0 |= (R.x >= p.drop_thr ? 1u : 0u) << e;
        m1 |= (R.y >= p.drop_thr ? 1u : 0u) << e;
        m2 |= (R.z >= p.drop_thr ? 1u : 0u) << e;
        m3 |= (R.w >= p.drop_thr ? 1u : 0u) << e;
      }
      // row r of the buffer: BM bits, 16-bit piece qg = columns 16 qg .. 16 qg + 15
      uint16_t *mb = reinterpret_cast<uint16_t *>(smem + C::OFF_MASK + buf * C::MASK_BUF) +
                     (4 * kq) * (C::BM / 16) + qg;
      mb[0] = (uint16_t)m0;
      mb[C::BM / 16] = (uint16_t)m1;
      mb[2 * (C::BM / 16)] = (uint16_t)m2;
      mb[3 * (C::BM / 16)] = (uint16_t)m3;
      mbar_arrive(bar(B_MFULL + buf));
      return true;
    };
    // dQ^T of step i of unit U (running step count gi): into registers, TMEM
    // released, then float32 reductions into the accumulator
    auto readout = [&](const Unit &U, int i, int gi) {
      if (!warp_wait_all(bar(B_DQFULL), gi & 1, wc)) return false;
      tc_fence_after();
      uint32_t v0[32], v1[32];
      if (live_rows) {
        tmem_ld32(src, v0);
        tmem_ld32(src + 32, v1);
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(bar(B_DQEMPTY));
      if (!live_rows) return true;
      const int h = step_head(U, i), q0 = step_qblk(U, i) * C::BM;
      const int nvalid = min(C::BM, p.Nq - q0);
      float *acc = p.dq_acc + (((size_t)(U.b * p.Hq + h)) * p.Nq + q0 + ch0 * 32) * C::D + t;
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (ch0 * 32 + c < nvalid) atomicAdd(acc + (size_t)c * C::D, __uint_as_float(v0[c]));
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (ch0 * 32 + 32 + c < nvalid) atomicAdd(acc + (size_t)(32 + c) * C::D, __uint_as_float(v1[c]));
      return true;
    };
    if constexpr (!DROP) {
      int gs = 0;
      for (int k = 0; ok; ++k) {
        ok = warp_wait_all(bar(B_UFULL + (k & 3)), (k >> 2) & 1, wc);
        if (!ok) break;
        const int u = s_queue[k & 3];
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_UEMPTY + (k & 3)));
        if (u < 0) break;
        const Unit U = decode(u);
        for (int i = 0; i < U.nsteps && ok; ++i) ok = readout(U, i, gs + i);
        gs += U.nsteps;
      }
    } else {
      Cursor cd{-1, 0, -1, false, Unit{}};   // dQ readout
      Cursor cm{-1, 0, -1, false, Unit{}};   // dropout mask, two steps ahead
      for (int pre = 0; pre < 2 && ok; ++pre) {
        ok = advance(cm);
        if (ok && !cm.end) ok = gen_mask(cm);
      }
      while (ok) {
        ok = advance(cd);
        if (!ok || cd.end) break;
        ok = readout(cd.U, cd.i, cd.g);
        if (ok) ok = advance(cm);
        if (ok && !cm.end) ok = gen_mask(cm);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_ALLOC);
  }
}

// c[b, hkv, :] = mean of the head's first min(Nk, 64) key rows, rounded to
// integers (f32).  One CTA per (batch, key/value head), one thread per column.
template <int D>
__global__ void bwd_center_kernel(const __nv_bfloat16 *__restrict__ k, float *__restrict__ cvec,
                                  int Nk, int *__restrict__ sched) {
  const int t = threadIdx.x;
  if (blockIdx.x == 0 && t == 0) *sched = 0;   // work counter of the dK/dV kernel
  const __nv_bfloat16 *kh = k + (size_t)blockIdx.x * Nk * D + t;
  const int nr = min(Nk, kCenterRows);
  float acc = 0.f;
  for (int j = 0; j < nr; ++j) acc += __bfloat162float(kh[(size_t)j * D]);
  cvec[(size_t)blockIdx.x * D + t] = rintf(acc / (float)nr);
}

// Per padded query row: D = sum_d dO * O and
// L2 = log2e * L - scale * log2e * (q . c) (rows past Nq: D = 0, L2 = +inf);
// zero the row of the dQ accumulator.  D / 8 lanes per row, each reading 16
// bytes of O, dO and Q (so a warp covers 32 * 8 / D rows).  A lane reads Q
// only where its 8 entries of c are not all zero: c is the key mean rounded
// to integers, zero for keys centred near 0, and the skipped products are
// exact zeros, so most calls read no Q at all (measured on B200 at causal B4
// H16 N4096 d128, centring and preprocess together: 64.5 -> 60.4 us).
template <int D>
__global__ void bwd_preprocess_kernel(const __nv_bfloat16 *__restrict__ q,
                                      const __nv_bfloat16 *__restrict__ o,
                                      const __nv_bfloat16 *__restrict__ dout,
                                      const float *__restrict__ lse,
                                      const float *__restrict__ cvec, float *__restrict__ dsum,
                                      float *__restrict__ l2, float *__restrict__ dq_acc,
                                      long long prow_total, int Nq, int npad, int Hq, int g,
                                      float scale_log2) {
  constexpr int LPR = D / 8;     // lanes per row
  constexpr int RPW = 32 / LPR;  // rows per warp
  const int lane = threadIdx.x & 31;
  const int l = lane % LPR;
  const long long prow = ((long long)blockIdx.x * 8 + (threadIdx.x >> 5)) * RPW + lane / LPR;
  const bool valid = prow < prow_total;
  const long long bh = valid ? prow / npad : 0;
  const int qi = valid ? (int)(prow - bh * npad) : 0;
  const bool live = valid && qi < Nq;
  const long long row = bh * Nq + qi;
  float sd = 0.f, sq = 0.f;
  if (live) {
    const int b = (int)(bh / Hq), h = (int)(bh % Hq);
    const float *cv = cvec + ((size_t)b * (Hq / g) + h / g) * D + l * 8;
    const uint4 ov = *reinterpret_cast<const uint4 *>(o + row * D + l * 8);
    const uint4 dv = *reinterpret_cast<const uint4 *>(dout + row * D + l * 8);
    const float4 c0 = *reinterpret_cast<const float4 *>(cv);
    const float4 c1 = *reinterpret_cast<const float4 *>(cv + 4);
    const bool need_q = c0.x != 0.f || c0.y != 0.f || c0.z != 0.f || c0.w != 0.f || c1.x != 0.f ||
                        c1.y != 0.f || c1.z != 0.f || c1.w != 0.f;
    const uint4 qv = need_q ? *reinterpret_cast<const uint4 *>(q + row * D + l * 8) : make_uint4(0, 0, 0, 0);
    const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w}, dw[4] = {dv.x, dv.y, dv.z, dv.w},
                   qw[4] = {qv.x, qv.y, qv.z, qv.w};
    const float cc[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ow[e]));
      const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&dw[e]));
      const float2 qq = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&qw[e]));
      sd = fmaf(a.x, c.x, sd);
      sd = fmaf(a.y, c.y, sd);
      sq = fmaf(qq.x, cc[2 * e], sq);
      sq = fmaf(qq.y, cc[2 * e + 1], sq);
    }
  }
#pragma unroll
  for (int off = LPR / 2; off > 0; off >>= 1) {
    sd += __shfl_xor_sync(0xffffffffu, sd, off);
    sq += __shfl_xor_sync(0xffffffffu, sq, off);
  }
  if (valid && l == 0) {
    dsum[prow] = live ? sd : 0.f;
    l2[prow] = live ? lse[row] * kLog2e - scale_log2 * sq : INFINITY;
  }
  if (live) {
    float4 *z = reinterpret_cast<float4 *>(dq_acc + row * D + l * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// dQ = bf16(scale * acc), 8 elements per thread.
__global__ void bwd_convert_kernel(const float *__restrict__ acc, __nv_bfloat16 *__restrict__ dq,
                                   long long n8, float scale) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = reinterpret_cast<const float4 *>(acc)[2 * i];
  const float4 c = reinterpret_cast<const float4 *>(acc)[2 * i + 1];
  uint4 out;
  out.x = pack_bf16x2(a.x * scale, a.y * scale);
  out.y = pack_bf16x2(a.z * scale, a.w * scale);
  out.z = pack_bf16x2(c.x * scale, c.y * scale);
  out.w = pack_bf16x2(c.z * scale, c.w * scale);
  reinterpret_cast<uint4 *>(dq)[i] = out;
}

bool make_map(CUtensorMap *m, const void *base, int rows_per_head, int heads, int d,
              int box_rows) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows_per_head, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)rows_per_head * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct WsPtrs {
  float *dsum, *l2, *cvec, *dq_acc;
  int *sched;
};
WsPtrs ws_ptrs(const AttnArgs &a) {
  char *w = (char *)a.ws;
  return {(float *)w, (float *)(w + ws_l2_offset(a.B, a.Hq, a.Nq)),
          (float *)(w + ws_c_offset(a.B, a.Hq, a.Nq)),
          (float *)(w + ws_dq_offset(a.B, a.Hq, a.Nq, a.d)),
          (int *)(w + ws_sched_offset(a.B, a.Hq, a.Nq, a.d))};
}

template <int D>
int run_prep(const AttnArgs &a) {
  const WsPtrs w = ws_ptrs(a);
  bwd_center_kernel<D><<<(unsigned)(a.B * a.Hkv), D, 0, a.stream>>>(
      (const __nv_bfloat16 *)a.k, w.cvec, a.Nk, w.sched);
  if (cudaGetLastError() != cudaSuccess) return 5;
  const int npad = (int)ws_npad(a.Nq);
  const long long prows = (long long)a.B * a.Hq * npad;
  constexpr int rows_per_block = 8 * (256 / D);   // 8 warps, 32 * 8 / D rows each
  bwd_preprocess_kernel<D><<<(unsigned)((prows + rows_per_block - 1) / rows_per_block), 256, 0,
                             a.stream>>>(
      (const __nv_bfloat16 *)a.q, (const __nv_bfloat16 *)a.o_in, (const __nv_bfloat16 *)a.dout,
      a.lse, w.cvec, w.dsum, w.l2, w.dq_acc, prows, a.Nq, npad, a.Hq, a.Hq / a.Hkv,
      a.scale * kLog2e);
  return cudaGetLastError() == cudaSuccess ? 0 : 5;
}

template <class C, bool WIDE>
int run_dkdv(const AttnArgs &a) {
  const WsPtrs w = ws_ptrs(a);
  CUtensorMap mq, mk, mv, mdo;
  if (!make_map(&mq, a.q, a.Nq, a.B * a.Hq, C::D, C::BM) ||
      !make_map(&mdo, a.dout, a.Nq, a.B * a.Hq, C::D, C::BM) ||
      !make_map(&mk, a.k, a.Nk, a.B * a.Hkv, C::D, C::BN) ||
      !make_map(&mv, a.v, a.Nk, a.B * a.Hkv, C::D, C::BN))
    return 5;
  BwdParams p;
  p.l2 = w.l2;
  p.dsum = w.dsum;
  p.cvec = w.cvec;
  p.dq_acc = w.dq_acc;
  p.sched = w.sched;
  p.dk = (__nv_bfloat16 *)a.dk;
  p.dv = (__nv_bfloat16 *)a.dv;
  p.Hq = a.Hq; p.Hkv = a.Hkv; p.Nq = a.Nq; p.Nk = a.Nk;
  p.npad = (int)ws_npad(a.Nq);
  p.nqb = (a.Nq + C::BM - 1) / C::BM;
  p.nkb = (a.Nk + C::BN - 1) / C::BN;
  p.BHkv = a.B * a.Hkv;
  {
    // causal unit order: groups of key/value heads whose f32 dQ accumulator
    // and Q, dO tiles (g query heads each) take about BWD_GROUP_BYTES, so the
    // reductions of a group stay in L2; inside a group the heaviest key
    // blocks first.  Non-causal units are all equal: head by head.
    const double per_kv_head = (double)(a.Hq / a.Hkv) * a.Nq * a.d * 8.0;
    const double hg = floor((double)BWD_GROUP_BYTES / per_kv_head);
    p.hg = !a.causal || hg < 1.0 ? 1 : (hg >= (double)p.BHkv ? p.BHkv : (int)hg);
  }
  p.scale = a.scale;
  p.scale_log2 = a.scale * kLog2e;
  p.causal = a.causal;
  p.err = a.err;
  const long long units = (long long)p.nkb * p.BHkv;
  if (units > 2147483647LL) return 2;
  p.drop_thr = a.drop_thr;
  p.seed_lo = (uint32_t)a.seed;
  p.seed_hi = (uint32_t)(a.seed >> 32);
  p.drop_off = (uint32_t)a.drop_offset;
  p.drop_scale = a.drop_scale;
  if constexpr (WIDE) {
    auto kern = bwd_wide_kernel<C, C::MASKGEN>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
        cudaSuccess)
      return 5;
    // persistent: one CTA per SM (at most one per unit)
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return 5;
    const long long grid = (BWD_PERSIST && units > sms) ? sms : units;
    kern<<<(unsigned)grid, C::THREADS, C::SMEM, a.stream>>>(mq, mk, mv, mdo, p);
  } else {
    auto kern = a.drop_thr != 0 ? bwd_kernel<C, true> : bwd_kernel<C, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
        cudaSuccess)
      return 5;
    // Persistent (one CTA per SM) when units are short, where a CTA's set-up
    // and epilogue weigh most; otherwise one CTA per unit, whose hardware
    // order balances the causal units' unequal lengths better than the
    // static snake.  Measured on B200 (dkdv, B*N = 32768, H16): N = 512
    // causal 1.334 -> 1.248 ms, N = 2048 causal 3.018 -> 2.798 ms, N = 8192
    // causal 9.61 -> 9.79 ms with the persistent grid.
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return 5;
    const bool persist = (long long)(a.Hq / a.Hkv) * p.nqb <= 32;
    const long long grid = persist && units > sms ? sms : units;
    kern<<<(unsigned)grid, kThreads, C::SMEM, a.stream>>>(mq, mk, mv, mdo, p);
  }
  return cudaGetLastError() == cudaSuccess ? 0 : 5;
}

int run_dq(const AttnArgs &a) {
  const WsPtrs w = ws_ptrs(a);
  const long long n8 = (long long)a.B * a.Hq * a.Nq * a.d / 8;
  bwd_convert_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, a.stream>>>(
      w.dq_acc, (__nv_bfloat16 *)a.dq, n8, a.scale);
  return cudaGetLastError() == cudaSuccess ? 0 : 5;
}

}  // namespace

int launch_bwd_prep_bf16(const AttnArgs &a) {
  switch (a.d) {
    case 64: return run_prep<64>(a);
    case 128: return run_prep<128>(a);
    case 256: return run_prep<256>(a);
    default: return 2;
  }
}


// d = 64 and 128: one pass with 128-row query blocks (bwd_wide_kernel).
// d = 256: dK and dV alone fill TMEM, so two passes of bwd_kernel (each CTA
// runs a static snake sequence of units, one unit per CTA when the grid has
// one CTA per unit).
// (bwd_kernel's single-pass mode, 64-row blocks in two TMEM sets, measured
// 8-11% slower than bwd_wide_kernel at d = 64 and 128.)
int launch_bwd_dkdv_bf16_sm100(const AttnArgs &a) {
  switch (a.d) {
    // dropout: the mask-generating instances (at d = 128 with a one-slot
    // Q/dO ring, which leaves room for the mask buffers)
    case 64:
      return a.drop_thr ? run_dkdv<BwdWideCfg<64, 4, true, true>, true>(a)
                        : run_dkdv<BwdWideCfg<64, 4, true>, true>(a);
    case 128:
      return a.drop_thr ? run_dkdv<BwdWideCfg<128, 1, false, true>, true>(a)
                        : run_dkdv<BwdWideCfg<128, 2, false>, true>(a);
    case 256: {
      int st = run_dkdv<BwdCfg<256, kDV, 64, 2, 2>, false>(a);
      return st ? st : run_dkdv<BwdCfg<256, kDKDQ, 64, 1, 1>, false>(a);
    }
    default: return 2;
  }
}

int launch_bwd_dq_bf16(const AttnArgs &a) { return run_dq(a); }

int launch_bwd_bf16_sm100(const AttnArgs &a) {
  int st = launch_bwd_prep_bf16(a);
  if (!st) st = launch_bwd_dkdv_bf16_sm100(a);
  if (!st) st = launch_bwd_dq_bf16(a);
  return st;
}

}  // namespace fa
