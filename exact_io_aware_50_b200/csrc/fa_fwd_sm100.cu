// fa_fwd_sm100.cu -- BF16 and E4M3 attention forward for sm_100a: TMA-fed
// shared-memory ring, tcgen05 MMA with TMEM accumulators, one softmax thread
// per query row.
//
// Method (FlashAttention blog, sections 2-4; CSDN FlashAttention-1 tutorial,
// section 3): Q is cut into 128-row tiles (outer loop, one or two tiles per
// CTA), K and V into 128-row blocks (inner loop).  For every block:
//     S = Q K_j^T                     tcgen05, bf16 x bf16 -> f32 in TMEM
//     m_new = max(m, rowmax(S*scale)) softmax thread of the row
//     P = exp(S*scale - m)            to shared memory (or TMEM) as bf16
//     l = e^{m_old - m} l + rowsum(P)
//     O~ = e^{m_old - m} O~ + P V_j   tcgen05, P and V from SMEM (or P from TMEM)
// and after the last block O = O~ / l, L = m + ln(l) (deferred
// normalisation, blog section 4.1).  The rescale of O~ is skipped while the
// running max has grown by less than 2^8 (in base-2 units): p values then stay
// below 256 and the final divide uses the same stale m, so the result is the
// same quantity (the wiki's FlashAttention-4 paragraph lists conditional
// rescaling; the exactness argument is the deferred-normalisation identity).
//
// Persistent CTAs (one per SM): each runs a fixed sequence of work units,
// keeping its TMEM, barriers and rings; the next unit's Q load and first S
// MMAs overlap the previous unit's epilogue.  Q is refilled once the last S
// of a unit has read it (barrier q_empty), O once the epilogue has read it
// out (o_empty).  Barrier phases follow running counters of key blocks and
// units across the sequence.
//
// Warp roles (10 warps, 320 threads, one CTA per SM):
//   warps 0-3  softmax + epilogue for Q tile 0 (thread = TMEM lane = row)
//   warps 4-7  softmax + epilogue for Q tile 1 (NT == 2)
//   warp  8    TMA producer (Q once, then K_j / V_j into STAGES-deep rings)
//   warp  9    MMA issuer
// The producer and MMA roles run in lane 0 alone (measured 6-8% faster on
// B200 than keeping the warp converged around each wait).
// Split-KV mode (inference shapes: few query blocks, long key range): work
// unit = (piece, batch, head, query block); each piece covers a contiguous
// range of the visible key blocks and writes its normalised partial output
// (float32) and log-sum-exp to a workspace; splitkv_combine_kernel merges the
// pieces with L = log sum_s exp(L_s), O = sum_s exp(L_s - L) O_s, the
// block-combination identity of the online softmax (blog section 2.2).  The
// causal mask may be bottom-right aligned there (key j hidden from query i
// when j > i + Nk - Nq).
//
// Dropout (DROP instances): the stored P keeps only the elements whose
// Philox4x32-10 word is >= floor(p 2^32) (one counter per four key columns of
// a row); the row sum uses the undropped P and the epilogue scales O by
// 1 / (1 - p).  The dropout instances hold one Q tile per CTA and warps
// 4-7 evaluate the counters for the key blocks ahead (FwdCfg MW); measured
// on B200 against the two-tile kernel whose softmax thread evaluated them
// (causal B4 H16 N4096 d128, p = 0.1): 0.80 -> 0.73 ms.
//
// CTA-pair instances (C::PAIR, fa_fwd_pair): clusters of two CTAs on one TPC
// run one unit sequence; the even CTA issues tcgen05 cta_group::2 MMAs (M =
// 256) for both, each CTA holding its own Q tiles, 64 of each K block's 128
// keys and d / 2 of each V block's columns (the two-CTA MMA that the wiki's
// FlashAttention-4 paragraph lists).  Loads of both CTAs complete on the
// leader's barriers, MMA commits arrive on both CTAs', and the softmax
// threads of both arrive on the leader's.  Measured on B200 20-35% slower
// than the single-CTA instances at d = 128 and 256 (the pair ties the two
// CTAs' per-block hand-offs together), so fa_fwd does not use it.
//
// E4M3 instances (C::F8): Q, K, V are one-byte OCP E4M3 codes with one
// dequantisation factor each.  S = Q K^T runs as tcgen05 kind::f8f6f4 (K = 32
// per instruction), the Q and K factors fold into the softmax scale, P is
// stored as e4m3 (one byte per key; four per TMEM column in the TMEM form)
// for the P V product (V MN-major, as in the bf16 path), and the V factor
// joins the final 1 / l.  P is stored as
// 2^4 * 2^(x - m) with the rescale threshold at 2^4, so stored values stay at
// or below 256 (e4m3 saturates at 448); the shift cancels in O / l and is
// taken out of L.  The wiki's FlashAttention-3 paragraph names FP8 as one of
// FA3's Hopper features and defines nothing further.
//
// Pipeline: the softmax thread reads S_t(j) out of TMEM and arrives on
// s_empty; the MMA issuer then starts S_t(j+1) in the same columns while
// block j's exponentials run.  P_t(j) goes to a K-major 128-byte-swizzled
// shared-memory tile once P_t(j-1) V_{j-1} has released it (p_empty, which
// also orders the rare O~ rescale after that MMA), and P_t(j) V_j runs
// SMEM x SMEM.  Issue order per block: S0(j+1), S1(j+1), PV0(j), PV1(j); the
// producer loads K one block ahead of V.  (Keeping P in TMEM over S_t's
// columns instead was measured slower on B200: at d = 128 the shared-memory
// form gained 2% with a 1-stage K/V ring against 2 stages, at d = 256 with
// one Q tile per CTA 23-35%.)
#include <math.h>

#include "common.cuh"
#include "cta_pair.cuh"
#include "launch.h"

namespace fa {
namespace {

constexpr int BM = 128;                 // query rows per tile (MMA M)
constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// ES: bytes per Q/K/V element, 2 for bf16, 1 for e4m3.  Tiles are laid out in
// bytes (128-byte swizzled rows), so an e4m3 d = 128 tile has the shape of a
// bf16 d = 64 one.
// P goes to shared memory, which frees S's TMEM columns as soon as the
// softmax has read them, so S(j+1) is issued while the softmax of block j
// still runs.
// MW (dropout instances with one Q tile per CTA): warps 4-7, which have no
// tile of their own, evaluate the Philox words of the dropout mask for the
// key blocks ahead and leave one bit per (query row, key) in a double-
// buffered array in shared memory, so the softmax thread tests bits instead
// of evaluating a Philox call per four keys.
// PAIR: a cluster of two CTAs shares each tile's MMAs (cta_group::2, M =
// 256): each CTA holds its own NT Q tiles, half of each K tile (64 of the
// 128 keys) and half of each V tile (D / 2 of the columns), so a K/V ring
// slot takes half the shared memory and half the load bytes per SM; the even
// CTA issues the MMAs for both.
// CSKIP (causal instances with two tiles, whole key range): a unit's last key
// block lies past tile 0's diagonal, so tile 0 stops one block early (its S
// and P V for that block are not issued; the block would only add zeros).
// Used up to 2048 keys: measured on B200 (d = 64 and 128) it gains 10-11% at
// 512 keys and 1-3% at 2048, is neutral at 4096 and loses 1-4% at 8192 and
// 16384, where tile 0 running a block ahead into the next unit offsets the
// two tiles' softmax phases.
template <int D_, int NT_, int BN_, int STAGES_, int ES_ = 2, bool MW_ = false, bool PAIR_ = false,
          bool CSKIP_ = false>
struct FwdCfg {
  static constexpr int D = D_, NT = NT_, BN = BN_, STAGES = STAGES_, ES = ES_;
  static constexpr bool MW = MW_, PAIR = PAIR_, CSKIP = CSKIP_;
  static constexpr bool F8 = ES == 1;
  static constexpr int DCH = D * ES / 128;                // 128-byte column chunks
  static constexpr int CH_ELEMS = 128 / ES;               // elements per chunk (TMA box width)
  static constexpr int MMA_K = 32 / ES;                   // K of one MMA: 32 bytes of a row
  static constexpr int S_STEPS = D / MMA_K;               // MMAs per S tile
  static constexpr int PV_STEPS = BN / MMA_K;             // MMAs per P V
  // P is stored as 2^P_SHIFT * 2^(x - m): for e4m3 that keeps the largest
  // stored value (2^(P_SHIFT + RESCALE)) inside the format's 448 and lifts
  // small values out of its subnormal range.
  static constexpr float P_SHIFT = F8 ? 4.f : 0.f;
  static constexpr float RESCALE = F8 ? 4.f : kRescaleThreshold;
  static constexpr int Q_CHUNK = BM * 128;                // bytes of one chunk of a Q tile
  static constexpr int KV_CHUNK = BN * 128;
  static constexpr int Q_TILE = Q_CHUNK * DCH;
  // this CTA's share of a K tile (rows) and of a V tile (128-byte column chunks)
  static constexpr int K_ROWS = PAIR ? BN / 2 : BN;
  static constexpr int V_DCH = PAIR ? DCH / 2 : DCH;
  static constexpr int K_CHUNK = K_ROWS * 128;
  static constexpr int K_TILE = K_CHUNK * DCH;
  static constexpr int V_TILE = KV_CHUNK * V_DCH;
  // query rows of one work unit (both CTAs of a pair)
  static constexpr int UROWS = (PAIR ? 2 : 1) * NT * 128;
  static constexpr int MMA_M = PAIR ? 256 : 128;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NT * Q_TILE;
  static constexpr int OFF_V = OFF_K + STAGES * K_TILE;
  // P tiles: [NT][BM rows][BN * ES bytes], K-major 128-byte swizzled chunks
  static constexpr int P_ROWB = BN * ES;
  static constexpr int P_CHUNK = BM * 128;
  static constexpr int P_TILE = P_CHUNK * (P_ROWB / 128);
  static constexpr int OFF_P = OFF_V + STAGES * V_TILE;
  static constexpr int MASK_BUF = BM * BN / 8;            // [MASK_NBUF][BM rows][BN bits]
  // d = 256 has room for one mask buffer only (and no alignment slack: the
  // dynamic shared window is 1024-byte aligned, checked at run time)
  static constexpr int MASK_NBUF = D >= 256 ? 1 : 2;
  static constexpr int SLACK = (MW && D >= 256) ? 0 : 1024;
  static constexpr int OFF_MASK = OFF_P + NT * P_TILE;
  static constexpr int OFF_BAR = OFF_MASK + (MW ? MASK_NBUF * MASK_BUF : 0);
  // barriers: q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[NT],
  // p_full[NT], o_full[NT], drain, q_empty, o_empty[NT], s_empty[NT] (S read
  // out of TMEM), p_empty[NT] (P V done with P), mask_full[2], mask_empty[2]
  static constexpr int NBAR = 1 + 4 * STAGES + 3 * NT + 1 + 1 + NT + 2 * NT + 4;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;     // tmem base slot, abort flag
  static constexpr int SMEM = OFF_MISC + 16 + SLACK;      // + alignment slack
  // TMEM columns
  static constexpr int TM_S = 0;                          // S_t at t*BN
  static constexpr int TM_O = NT * BN;                    // O_t at TM_O + t*D
  static constexpr int TM_COLS_USED = NT * (BN + D);
  static constexpr int TM_ALLOC = 512;
  static_assert(TM_COLS_USED <= TM_ALLOC, "TMEM budget");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(BN == 128, "softmax path assumes 128 columns per block");
  static_assert(ES == 1 || ES == 2, "bf16 or e4m3 operands");
  static_assert(D * ES % 128 == 0, "whole 128-byte rows per chunk");
  static_assert(!MW || (NT == 1 && ES == 2 && BN == 128), "mask warps: one bf16 tile per CTA");
  static_assert(!PAIR || (!MW && ES == 2 && DCH % 2 == 0), "pairs: bf16, d = 128 or 256, no dropout");
  static_assert(!CSKIP || (NT == 2 && !PAIR && !MW), "tile-0 early stop: two tiles per CTA");
};

struct FwdParams {
  float *o_lse;      // lse output
  __nv_bfloat16 *o;  // O output
  int Hq, Hkv, Nq, Nk, nqb;  // nqb = query blocks (of NT*128 rows) per head
  int BH;            // B * Hq
  float scale_log2;  // scale * log2(e)
  int causal;
  int causal_off;    // causal: key j hidden from query i when j > i + causal_off
  int splits;        // pieces of the key range per query block (1: plain forward)
  int hg;            // causal: heads per group of the unit order (BH: one group)
  float *o_part;     // splits > 1: [splits][B*Hq][Nq][D] normalised partial O
  float *l_part;     // splits > 1: [splits][B*Hq][Nq] partial log-sum-exp (natural log)
  // dropout on P (DROP kernels): keep when the Philox word >= drop_thr; kept
  // values are scaled by 1 / (1 - p) (o_scale) in the epilogue
  uint32_t drop_thr, seed_lo, seed_hi, drop_off;
  float o_scale;     // epilogue factor on O: 1 / (1 - p) with dropout, the V descale for e4m3
  unsigned *err;
};

template <class C, bool DROP>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  static_assert(!(DROP && C::F8), "dropout is built for the bf16 forward only");
  static_assert(DROP == C::MW, "dropout instances take their mask from the mask warps");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (C::SLACK == 0 && (smem_u32(smem_raw) & 1023u)) {
    if (threadIdx.x == 0) atomicOr(p.err, kErrConfig);
    return;
  }
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t *bars = (uint64_t *)(smem + C::OFF_BAR);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const int B_QFULL = 0;
  const int B_KFULL = 1, B_KEMPTY = 1 + C::STAGES, B_VFULL = 1 + 2 * C::STAGES,
            B_VEMPTY = 1 + 3 * C::STAGES;
  const int B_SFULL = 1 + 4 * C::STAGES, B_PFULL = B_SFULL + C::NT, B_OFULL = B_PFULL + C::NT;
  const int B_DRAIN = B_OFULL + C::NT;
  const int B_QEMPTY = B_DRAIN + 1, B_OEMPTY = B_DRAIN + 2;
  const int B_SEMPTY = B_OEMPTY + C::NT, B_PEMPTY = B_SEMPTY + C::NT;
  const int B_MFULL = B_PEMPTY + C::NT, B_MEMPTY = B_MFULL + 2;
  static_assert(!C::MW || DROP, "mask warps only in dropout instances");
  uint32_t *tmem_slot = (uint32_t *)(smem + C::OFF_MISC);
  volatile int *abort_flag = (volatile int *)(smem + C::OFF_MISC + 4);

  const int warp = warp_id_uniform();
  const int lane = threadIdx.x & 31;
  // CTA pairs: the pair runs one unit sequence; its rank-0 CTA (the leader)
  // issues the MMAs and owns the barriers they wait on.
  const uint32_t rank = C::PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  // cluster address of the leader's barrier i (pairs)
  auto lbar = [&](int i) { return mapa_shared(bar(i), 0); };
  // arrive on a barrier the MMA issuer waits for
  auto arrive_mma = [&](int i) {
    if constexpr (C::PAIR) mbar_arrive_cluster(lbar(i));
    else mbar_arrive(bar(i));
  };

  // Persistent CTAs (or pairs): round k gives CTA c unit k*G + c (k even)
  // or k*G + G-1-c (k odd), G = gridDim.x (pairs: G pairs, c the pair's
  // index).  Unit order:
  // causal, the heaviest query blocks of every head first; otherwise head by
  // head, so the K and V tiles a wave reads are those of a few heads and stay
  // in L2.  Split-KV: the piece index is the slowest-varying part.
  const int per_piece = p.nqb * p.BH;
  const int total_units = per_piece * p.splits;
  const int G = (int)gridDim.x / (C::PAIR ? 2 : 1);
  const int cid = (int)blockIdx.x / (C::PAIR ? 2 : 1);
  auto unit_at = [&](int k) { return k * G + ((k & 1) ? G - 1 - cid : cid); };
  struct Unit {
    int piece, bh, bh_kv, q_start, j0, nkb;
    int nkb0;   // key blocks of Q tile 0 (CSKIP: one fewer when its diagonal ends earlier)
  };
  auto decode = [&](int u) {
    Unit U;
    U.piece = u / per_piece;
    const int v = u % per_piece;
    int qblk;
    if (p.causal) {
      // heaviest query blocks first, inside groups of hg heads taken one
      // group after the other (the last group may be smaller)
      const int grp = v / (p.nqb * p.hg);
      const int w = v - grp * p.nqb * p.hg;
      const int gsize = min(p.hg, p.BH - grp * p.hg);
      qblk = p.nqb - 1 - w / gsize;
      U.bh = grp * p.hg + w % gsize;
    } else {
      qblk = v % p.nqb;
      U.bh = v / p.nqb;
    }
    const int b = U.bh / p.Hq, h = U.bh % p.Hq;
    U.bh_kv = b * p.Hkv + h / (p.Hq / p.Hkv);
    U.q_start = qblk * C::UROWS;
    const int nkb_all = (p.Nk + C::BN - 1) / C::BN;
    const int nkb_vis = p.causal
                            ? min(nkb_all, (U.q_start + C::UROWS + p.causal_off + C::BN - 1) / C::BN)
                            : nkb_all;
    // key blocks [j0, j0 + nkb) of this piece
    const int per_split = (nkb_vis + p.splits - 1) / p.splits;
    U.j0 = min(nkb_vis, U.piece * per_split);
    U.nkb = min(nkb_vis, U.j0 + per_split) - U.j0;
    U.nkb0 = U.nkb;
    if constexpr (C::CSKIP)   // causal, one piece (the launcher checks)
      U.nkb0 = min(U.nkb, (U.q_start + BM + p.causal_off + C::BN - 1) / C::BN);
    return U;
  };
  auto nkb_of = [&](const Unit &U, int t) { return (C::CSKIP && t == 0) ? U.nkb0 : U.nkb; };
  // first query row of this CTA's tile t of unit U
  auto tile_row0 = [&](const Unit &U, int t) { return U.q_start + ((int)rank * C::NT + t) * BM; };

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    mbar_init(bar(B_QEMPTY), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_KEMPTY + s), 1);
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_VEMPTY + s), 1);
    }
    for (int t = 0; t < C::NT; ++t) {
      mbar_init(bar(B_SFULL + t), 1);
      // arrivals of the softmax threads: both CTAs' in a pair
      mbar_init(bar(B_PFULL + t), (C::PAIR ? 2 : 1) * BM);
      mbar_init(bar(B_OFULL + t), 1);
      mbar_init(bar(B_OEMPTY + t), (C::PAIR ? 2 : 1) * BM);
      mbar_init(bar(B_SEMPTY + t), (C::PAIR ? 2 : 1) * BM);
      mbar_init(bar(B_PEMPTY + t), 1);
    }
    mbar_init(bar(B_DRAIN), 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(B_MFULL + x), BM);    // the mask threads wrote their rows
      mbar_init(bar(B_MEMPTY + x), BM);   // the softmax threads read theirs
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    // pairs: warp 0 of both CTAs allocates the same columns in each
    if constexpr (C::PAIR) {
      tmem_alloc_pair(smem_u32(tmem_slot), C::TM_ALLOC);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), C::TM_ALLOC);
      tmem_relinquish();
    }
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  tc_fence_before();
  // pairs: the peer's first arrivals on the leader's barriers come after this
  if constexpr (C::PAIR) cluster_sync_all();
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  WaitCtx wc{p.err, abort_flag, kWaitLimitNs};

  // Ring positions run on across units: g counts key blocks, uq units with
  // work (barrier phases are these counters' parities).
  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    // The whole role runs in lane 0; the other lanes wait at the end.
    if (lane == 0) {
      int last_k_phase[C::STAGES], last_v_phase[C::STAGES];
      for (int s = 0; s < C::STAGES; ++s) last_k_phase[s] = last_v_phase[s] = -1;
      int last_q_phase = -1;
      bool ok = true;
      int g = 0, uq = 0;
      // A tile load completing on full-barrier fb: pairs load this CTA's half
      // and complete on the leader's barrier, where the leader alone has
      // announced both halves' bytes.
      auto load = [&](uint32_t dst, const CUtensorMap *m, int fb, int c0, int c1, int c2) {
        if constexpr (C::PAIR) tma_load_3d_pair(dst, m, lbar(fb), c0, c1, c2);
        else tma_load_3d(dst, m, bar(fb), c0, c1, c2);
      };
      constexpr uint32_t HALVES = C::PAIR ? 2 : 1;
      for (int k = 0; ok && k * G < total_units; ++k) {
        // snake order: even rounds ascending, odd rounds descending, so the
        // heavy-first unit list pairs heavy with light units on each CTA
        const int u = unit_at(k);
        if (u >= total_units) continue;
        const Unit U = decode(u);
        if (U.nkb == 0) continue;
        // the previous unit's S MMAs must be done with the Q tiles
        ok = bounded_wait(bar(B_QEMPTY), (uq & 1) ^ 1, wc);
        if (!ok) break;
        if (leader) mbar_arrive_expect_tx(bar(B_QFULL), HALVES * C::NT * C::Q_TILE);
        for (int t = 0; t < C::NT; ++t)
          for (int c = 0; c < C::DCH; ++c)
            load(sbase + C::OFF_Q + t * C::Q_TILE + c * C::Q_CHUNK, &tmQ, B_QFULL,
                 c * C::CH_ELEMS, tile_row0(U, t), U.bh);
        last_q_phase = uq & 1;
        // K: this CTA's K_ROWS keys of the block, all columns
        auto load_k = [&](int j) {
          const int s = (g + j) % C::STAGES;
          const uint32_t ph = ((g + j) / C::STAGES) & 1;
          if (!bounded_wait(bar(B_KEMPTY + s), ph ^ 1, wc)) return false;
          if (leader) mbar_arrive_expect_tx(bar(B_KFULL + s), HALVES * C::K_TILE);
          for (int c = 0; c < C::DCH; ++c)
            load(sbase + C::OFF_K + s * C::K_TILE + c * C::K_CHUNK, &tmK, B_KFULL + s,
                 c * C::CH_ELEMS, (U.j0 + j) * C::BN + (int)rank * C::K_ROWS, U.bh_kv);
          last_k_phase[s] = ph;
          return true;
        };
        // V: all keys of the block, this CTA's V_DCH column chunks
        auto load_v = [&](int j) {
          const int s = (g + j) % C::STAGES;
          const uint32_t ph = ((g + j) / C::STAGES) & 1;
          if (!bounded_wait(bar(B_VEMPTY + s), ph ^ 1, wc)) return false;
          if (leader) mbar_arrive_expect_tx(bar(B_VFULL + s), HALVES * C::V_TILE);
          for (int c = 0; c < C::V_DCH; ++c)
            load(sbase + C::OFF_V + s * C::V_TILE + c * C::KV_CHUNK, &tmV, B_VFULL + s,
                 ((int)rank * C::V_DCH + c) * C::CH_ELEMS, (U.j0 + j) * C::BN, U.bh_kv);
          last_v_phase[s] = ph;
          return true;
        };
        // Loads follow the MMA issuer's order of use (S runs a block ahead):
        // K_0, K_1, V_0, K_2, V_1, ...
        ok = load_k(0);
        for (int j = 0; j < U.nkb && ok; ++j) {
          if (j + 1 < U.nkb) ok = load_k(j + 1);
          if (ok) ok = load_v(j);
        }
        g += U.nkb;
        ++uq;
      }
      if (!ok && leader) {
        // Drain: let every copy this role issued land before the CTA exits.
        // (A pair's copies complete on the leader's barriers: the leader
        // drains them, the peer cannot observe its own.)
        if (last_q_phase >= 0) (void)drain_wait(bar(B_QFULL), last_q_phase, p.err, kWaitLimitNs);
        for (int s = 0; s < C::STAGES; ++s) {
          if (last_k_phase[s] >= 0) (void)drain_wait(bar(B_KFULL + s), last_k_phase[s], p.err, kWaitLimitNs);
          if (last_v_phase[s] >= 0) (void)drain_wait(bar(B_VFULL + s), last_v_phase[s], p.err, kWaitLimitNs);
        }
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // pairs: M = 256 (each CTA's 128 rows), N the whole block / head dim
    constexpr uint32_t IDESC_S =
        C::F8 ? idesc_e4m3(BM, C::BN, 0, 0) : idesc_bf16(C::MMA_M, C::BN, 0, 0);
    constexpr uint32_t IDESC_PV =
        C::F8 ? idesc_e4m3(BM, C::D, 0, 1) : idesc_bf16(C::MMA_M, C::D, 0, 1);
    auto mma16 = [&](uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
      if constexpr (C::PAIR) mma_ss_pair(d, a, b, idesc, acc);
      else mma_ss(d, a, b, idesc, acc);
    };
    // MMA completion: pairs arrive on the barrier in both CTAs
    auto commit = [&](int i) {
      if constexpr (C::PAIR) mma_commit_pair_both(bar(i));
      else mma_commit(bar(i));
    };
    // barriers the peer's threads arrive on (pairs) need cluster-scope acquire
    auto wait = [&](int i, uint32_t ph) {
      if constexpr (C::PAIR) return bounded_wait_cluster(bar(i), ph, wc);
      else return bounded_wait(bar(i), ph, wc);
    };
    // Descriptors are built once; each MMA offsets a base descriptor.
    const uint64_t dq0 = sw128_desc(sbase + C::OFF_Q, 16, 1024);
    const uint64_t dk0 = sw128_desc(sbase + C::OFF_K, 16, 1024);
    const uint64_t dv0 = sw128_desc(sbase + C::OFF_V, C::KV_CHUNK, 1024);
    auto issue_S = [&](int t, int s) {
      const uint64_t qa = desc_add(dq0, t * C::Q_TILE);
      const uint64_t kb = desc_add(dk0, s * C::K_TILE);
#pragma unroll
      for (int kk = 0; kk < C::S_STEPS; ++kk) {
        const uint32_t off = (kk >> 2) * C::Q_CHUNK + (kk & 3) * 32;
        const uint32_t offk = (kk >> 2) * C::K_CHUNK + (kk & 3) * 32;
        if constexpr (C::F8)
          mma_ss_f8(tmem + C::TM_S + t * C::BN, desc_add(qa, off), desc_add(kb, offk), IDESC_S,
                    kk > 0);
        else
          mma16(tmem + C::TM_S + t * C::BN, desc_add(qa, off), desc_add(kb, offk), IDESC_S,
                kk > 0);
      }
    };
    const uint64_t dp0 = sw128_desc(sbase + C::OFF_P, 16, 1024);
    auto issue_PV = [&](int t, int s, bool first) {
      const uint64_t vb = desc_add(dv0, s * C::V_TILE);
      const uint64_t pa = desc_add(dp0, t * C::P_TILE);
#pragma unroll
      for (int kk = 0; kk < C::PV_STEPS; ++kk) {
        // 32 bytes of a K-major shared-memory P row (MMA_K keys); MMA_K rows
        // of the MN-major V tile
        const uint32_t offp = (kk >> 2) * C::P_CHUNK + (kk & 3) * 32;
        if constexpr (C::F8)
          mma_ss_f8(tmem + C::TM_O + t * C::D, desc_add(pa, offp), desc_add(vb, kk * C::MMA_K * 128),
                    IDESC_PV, (!first) || kk > 0);
        else
          mma16(tmem + C::TM_O + t * C::D, desc_add(pa, offp), desc_add(vb, kk * C::MMA_K * 128),
                IDESC_PV, (!first) || kk > 0);
      }
    };
    // The whole role runs in lane 0 (of the leader, in a pair); the other
    // lanes wait at the end.
    if (lane == 0 && leader) {
      bool ok = true;
      int g = 0, uq = 0;
      // CSKIP: key blocks each tile has processed (its barriers' phases)
      int gt[C::NT];
      for (int t = 0; t < C::NT; ++t) gt[t] = 0;
      auto tile_phase = [&](int t, int j) {
        return (uint32_t)((C::CSKIP ? gt[t] + j : g + j) & 1);
      };
      for (int k = 0; ok && k * G < total_units; ++k) {
        // snake order: even rounds ascending, odd rounds descending, so the
        // heavy-first unit list pairs heavy with light units on each CTA
        const int u = unit_at(k);
        if (u >= total_units) continue;
        const Unit U = decode(u);
        if (U.nkb == 0) continue;
        ok = wait(B_QFULL, uq & 1);
        if (ok) ok = wait(B_KFULL + g % C::STAGES, (g / C::STAGES) & 1);
        if (!ok) break;
        tc_fence_after();
        for (int t = 0; t < C::NT; ++t) {
          issue_S(t, g % C::STAGES);
          commit(B_SFULL + t);
        }
        commit(B_KEMPTY + g % C::STAGES);
        if (U.nkb == 1) commit(B_QEMPTY);   // last S of the unit issued
        // S_t(j+1) as soon as the softmax has read S_t(j); P_t(j) V_j once
        // P_t(j) is in shared memory.
        for (int j = 0; j < U.nkb && ok; ++j) {
          const int gj = g + j;
          const int s = gj % C::STAGES;
          const uint32_t ph = (gj / C::STAGES) & 1;
          if (j + 1 < U.nkb) {
            const int s1 = (gj + 1) % C::STAGES;
            ok = wait(B_KFULL + s1, ((gj + 1) / C::STAGES) & 1);
            for (int t = 0; t < C::NT && ok; ++t) {
              if (C::CSKIP && j + 1 >= nkb_of(U, t)) continue;
              ok = wait(B_SEMPTY + t, tile_phase(t, j));
              if (!ok) break;
              tc_fence_after();
              issue_S(t, s1);
              commit(B_SFULL + t);
            }
            if (!ok) break;
            commit(B_KEMPTY + s1);
            if (j + 2 == U.nkb) commit(B_QEMPTY);   // last S of the unit
          }
          ok = wait(B_VFULL + s, ph);
          for (int t = 0; t < C::NT && ok; ++t) {
            if (C::CSKIP && j >= nkb_of(U, t)) continue;
            ok = wait(B_PFULL + t, tile_phase(t, j));
            if (ok && j == 0 && uq > 0)   // the previous unit's epilogue has read O_t
              ok = wait(B_OEMPTY + t, (uq - 1) & 1);
            if (!ok) break;
            tc_fence_after();
            issue_PV(t, s, j == 0);
            commit(B_PEMPTY + t);
            if (j + 1 == nkb_of(U, t)) commit(B_OFULL + t);
          }
          if (ok) commit(B_VEMPTY + s);
        }
        g += U.nkb;
        if constexpr (C::CSKIP)
          for (int t = 0; t < C::NT; ++t) gt[t] += nkb_of(U, t);
        ++uq;
      }
      if (!ok) {
        // Drain: every MMA issued so far must finish before TMEM is freed.
        if constexpr (C::PAIR) mma_commit_pair_local(bar(B_DRAIN));
        else mma_commit(bar(B_DRAIN));
        (void)drain_wait(bar(B_DRAIN), 0, p.err, kWaitLimitNs);
      }
    }
    __syncwarp();
  } else if (warp < 4 * C::NT) {
    // ------------------------------------------------------------ softmax
    const int t = warp >> 2;                  // Q tile of this warpgroup
    const int r = threadIdx.x & 127;          // row within the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::TM_S + t * C::BN;
    const uint32_t tO = tmem + lane_off + C::TM_O + t * C::D;
    bool ok = true;
    int g = 0, uq = 0;
    for (int k = 0; ok && k * G < total_units; ++k) {
        // snake order: even rounds ascending, odd rounds descending, so the
        // heavy-first unit list pairs heavy with light units on each CTA
        const int u = unit_at(k);
        if (u >= total_units) continue;
      const Unit U = decode(u);
      const int bh = U.bh;
      const int row = tile_row0(U, t) + r;     // query row
      if (U.nkb == 0) {
        // An empty piece (only in split mode): its rows see no key here.
        if (row < p.Nq) {
          const size_t prow = ((size_t)U.piece * p.BH + bh) * p.Nq + row;
          p.l_part[prow] = -INFINITY;
          float4 *orow = reinterpret_cast<float4 *>(p.o_part + prow * C::D);
          for (int e = 0; e < C::D / 4; ++e) orow[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        continue;
      }
      const int row_lo = tile_row0(U, t);
      const int nkb_t = nkb_of(U, t);   // g counts this tile's key blocks
      // keys [0, limit) visible
      const int limit_row = p.causal ? min(p.Nk, row + 1 + p.causal_off) : p.Nk;
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < nkb_t; ++j) {
        ok = warp_wait_all(bar(B_SFULL + t), (g + j) & 1, wc);
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[C::BN];
#pragma unroll
        for (int c = 0; c < C::BN / 32; ++c)
          tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
        tmem_wait_ld();
        // S_t is in registers: its TMEM columns may take S_t(j+1)
        tc_fence_before();
        arrive_mma(B_SEMPTY + t);
        float *s = reinterpret_cast<float *>(sr);
        const int col_lo = (U.j0 + j) * C::BN;
        // dropout with mask warps: bit 32 c + b of this row's 128 = key
        // col_lo + 32 c + b kept
        uint32_t mbits[4] = {0u, 0u, 0u, 0u};
        if constexpr (C::MW) {
          const int gj = g + j;
          const int mbuf = gj % C::MASK_NBUF;
          ok = warp_wait_all(bar(B_MFULL + mbuf), (gj / C::MASK_NBUF) & 1, wc);
          if (!ok) break;
          const uint4 mb = *reinterpret_cast<const uint4 *>(smem + C::OFF_MASK + mbuf * C::MASK_BUF +
                                                            r * (C::BN / 8));
          mbits[0] = mb.x; mbits[1] = mb.y; mbits[2] = mb.z; mbits[3] = mb.w;
          mbar_arrive(bar(B_MEMPTY + mbuf));
        }
        const bool need_mask =
            (col_lo + C::BN > p.Nk) || (p.causal && col_lo + C::BN - 1 > row_lo + p.causal_off);
        if (need_mask) {
          const int lim = limit_row - col_lo;
  #pragma unroll
          for (int c = 0; c < C::BN; ++c) s[c] = (c < lim) ? s[c] : -INFINITY;
        }
        // row max: eight independent partial maxima, then a small tree
        float mp[8];
  #pragma unroll
        for (int u = 0; u < 8; ++u) mp[u] = s[u];
  #pragma unroll
        for (int c = 8; c < C::BN; c += 8)
  #pragma unroll
          for (int u = 0; u < 8; ++u) mp[u] = fmaxf(mp[u], s[c + u]);
        const float mx = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                               fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
        const float m_new = fmaxf(m_run, mx * p.scale_log2);
        bool rescale = false;
        float alpha = 1.f;
        if (j == 0) {
          m_run = m_new;
        } else if (__any_sync(0xffffffffu, m_new - m_run > C::RESCALE)) {
          rescale = true;
          alpha = fast_exp2(m_run - m_new);
          m_run = m_new;
        }
        const float m_use = ((m_run == -INFINITY) ? 0.f : m_run) - C::P_SHIFT;
        // p = 2^(s * scale * log2e - m) on MUFU; row sum in four independent
        // partials over the undropped p; with dropout, the stored P keeps
        // only the columns whose Philox word is >= drop_thr (one Philox call
        // per four key columns)
        float rs[4] = {0.f, 0.f, 0.f, 0.f};
        // row r of the K-major shared-memory P tile (16-byte units swizzled
        // by r mod 8); written chunk by chunk once P_t(j-1) V_{j-1} is done
        // with it (waited before the first store: by then the MMA has had the
        // row maximum and 32 exponentials' time)
        const uint32_t prow = sbase + C::OFF_P + t * C::P_TILE + r * 128;
        const int r7 = r & 7;
  #pragma unroll
        for (int c = 0; c < C::BN / 32; ++c) {
          uint32_t pk[16];
  #pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float x0 = fmaf(s[c * 32 + 2 * e], p.scale_log2, -m_use);
            const float x1 = fmaf(s[c * 32 + 2 * e + 1], p.scale_log2, -m_use);
            const float p0 = fast_exp2(x0);
            const float p1 = fast_exp2(x1);
            rs[e & 3] += p0 + p1;
            if (DROP) {
              const uint32_t mw = mbits[c];
              pk[e] = pack_bf16x2(((mw >> (2 * e)) & 1u) ? p0 : 0.f, ((mw >> (2 * e + 1)) & 1u) ? p1 : 0.f);
            } else if constexpr (C::F8) {
              // four e4m3 codes per 32-bit word: keys 2e, 2e + 1 in the low
              // half of word e / 2 for even e, in the high half for odd e
              const uint32_t h = pack_e4m3x2(p0, p1);
              pk[e >> 1] = (e & 1) ? (pk[e >> 1] | (h << 16)) : h;
            } else {
              pk[e] = pack_bf16x2(p0, p1);
            }
          }
          if (c == 0 && j > 0) {
            ok = warp_wait_all(bar(B_PEMPTY + t), (g + j - 1) & 1, wc);
            tc_fence_after();
          }
          if (ok) {
  #pragma unroll
            for (int i = 0; i < 2 * C::ES; ++i) {   // 32 keys = 2 * ES 16-byte units
              const int b = c * 32 * C::ES + 16 * i;
              const int u = (b >> 4) & 7;
              st_shared_v4(prow + (b >> 7) * C::P_CHUNK + ((u ^ r7) << 4), pk[4 * i], pk[4 * i + 1],
                           pk[4 * i + 2], pk[4 * i + 3]);
            }
          }
        }
        const float rowsum = (rs[0] + rs[1]) + (rs[2] + rs[3]);
        l_run = l_run * alpha + rowsum;
        if (!ok) break;
        fence_proxy_async_smem();   // P stores visible to the tensor core
        // (P_t(j-1) V_{j-1}, which accumulates into O_t, was waited for above,
        // so O_t may be rescaled)
        if (rescale) {
  #pragma unroll 1
          for (int c = 0; c < C::D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(tO + c * 32, ov);
            tmem_wait_ld();
  #pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st32(tO + c * 32, ov);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        arrive_mma(B_PFULL + t);
      }
      // ---------------------------------------------------------- epilogue
      if (ok) ok = warp_wait_all(bar(B_OFULL + t), uq & 1, wc);
      if (ok && p.splits > 1) {
        // normalised partial output and log-sum-exp of this piece; a row whose
        // keys in the piece are all hidden has l = 0: O_s = 0, L_s = -inf
        tc_fence_after();
        const bool empty = !(l_run > 0.f);
        const float inv_l = empty ? 0.f : 1.f / l_run;
        const bool live = row < p.Nq;
        const size_t prow = ((size_t)U.piece * p.BH + bh) * p.Nq + (live ? row : 0);
        float4 *orow = reinterpret_cast<float4 *>(p.o_part + prow * C::D);
  #pragma unroll 1
        for (int c = 0; c < C::D / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(tO + c * 32, ov);
          tmem_wait_ld();
          if (live) {
  #pragma unroll
            for (int e = 0; e < 8; ++e)
              orow[c * 8 + e] = make_float4(__uint_as_float(ov[4 * e]) * inv_l,
                                            __uint_as_float(ov[4 * e + 1]) * inv_l,
                                            __uint_as_float(ov[4 * e + 2]) * inv_l,
                                            __uint_as_float(ov[4 * e + 3]) * inv_l);
          }
        }
        tc_fence_before();
        arrive_mma(B_OEMPTY + t);   // O_t read out: the next unit may overwrite it
        if (live)
          p.l_part[prow] =
              empty ? -INFINITY : (m_run + __log2f(l_run) - C::P_SHIFT) * 0.69314718055994531f;
      } else if (ok) {
        tc_fence_after();
        const float inv_l = p.o_scale / l_run;
        const bool live = row < p.Nq;
        __nv_bfloat16 *orow = p.o + ((size_t)bh * p.Nq + (live ? row : 0)) * C::D;
  #pragma unroll 1
        for (int c = 0; c < C::D / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(tO + c * 32, ov);
          tmem_wait_ld();
          uint32_t pk[16];
  #pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(ov[2 * e]) * inv_l,
                                __uint_as_float(ov[2 * e + 1]) * inv_l);
          if (live) {
            uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
  #pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
          }
        }
        tc_fence_before();
        arrive_mma(B_OEMPTY + t);   // O_t read out: the next unit may overwrite it
        if (live)
          p.o_lse[(size_t)bh * p.Nq + row] =
              (m_run + __log2f(l_run) - C::P_SHIFT) * 0.69314718055994531f;
      }
      g += nkb_t;
      ++uq;
    }
  } else if (C::MW && warp < 8) {
    // ------------------------------------------------------------ mask
    // Thread r evaluates the dropout mask of query row r of the tile for the
    // key blocks in order, up to two blocks ahead of the softmax: counter
    // (key / 4, query row, b*Hq + h, offset), word key % 4 - the words the
    // backward regenerates - into bits 4 k .. 4 k + 3 of the row's 128.
    const int r = threadIdx.x - 4 * 32;
    bool ok = true;
    int g = 0;
    for (int k = 0; ok && k * G < total_units; ++k) {
      const int u = unit_at(k);
      if (u >= total_units) continue;
      const Unit U = decode(u);
      const uint32_t row = (uint32_t)(U.q_start + r);
      for (int j = 0; j < U.nkb && ok; ++j) {
        const int gj = g + j;
        const int mbuf = gj % C::MASK_NBUF;
        ok = warp_wait_all(bar(B_MEMPTY + mbuf), ((gj / C::MASK_NBUF) & 1) ^ 1, wc);
        if (!ok) break;
        const uint32_t c0 = (uint32_t)((U.j0 + j) * C::BN) >> 2;
        uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          // four calls in flight per thread (measured on B200 against 1, 2
          // and 8: causal B4 H16 N4096 d128, p = 0.1, forward 0.92 / 0.74 /
          // 0.73 / 1.05 ms for 1 / 2 / 4 / 8)
#pragma unroll 4
          for (int kk = 0; kk < 8; ++kk) {
            const uint4 R = philox4x32_10(c0 + 8 * q4 + kk, row, (uint32_t)U.bh, p.drop_off, p.seed_lo,
                                          p.seed_hi);
            const uint32_t nib = (R.x >= p.drop_thr ? 1u : 0u) | (R.y >= p.drop_thr ? 2u : 0u) |
                                 (R.z >= p.drop_thr ? 4u : 0u) | (R.w >= p.drop_thr ? 8u : 0u);
            w[q4] |= nib << (4 * kk);
          }
        }
        st_shared_v4(sbase + C::OFF_MASK + mbuf * C::MASK_BUF + r * (C::BN / 8), w[0], w[1], w[2], w[3]);
        mbar_arrive(bar(B_MFULL + mbuf));
      }
      g += U.nkb;
    }
  }

  tc_fence_before();
  // pairs: neither CTA leaves (or frees its TMEM) while the other may still
  // arrive on its barriers or the leader's MMAs may still use it
  if constexpr (C::PAIR) cluster_sync_all();
  else __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    if constexpr (C::PAIR) tmem_dealloc_pair(tmem, C::TM_ALLOC);
    else tmem_dealloc(tmem, C::TM_ALLOC);
  }
}

// [heads][rows][d] tensor of `es`-byte elements (2: bf16, 1: e4m3 bytes);
// box = one 128-byte chunk of box_rows rows, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, int rows_per_head, int heads, int d,
              int box_rows, int es = 2) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows_per_head, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)d * es, (cuuint64_t)rows_per_head * d * es};
  cuuint32_t box[3] = {(cuuint32_t)(128 / es), (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType dt = es == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return enc(m, dt, 3, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <class C>
int run_fwd(const AttnArgs &a) {
  CUtensorMap mq, mk, mv;
  if (C::F8 && (a.drop_thr != 0 || a.splits > 1)) return 2;   // e4m3: plain forward only
  if (!make_map(&mq, a.q, a.Nq, a.B * a.Hq, C::D, BM, C::ES) ||
      !make_map(&mk, a.k, a.Nk, a.B * a.Hkv, C::D, C::K_ROWS, C::ES) ||
      !make_map(&mv, a.v, a.Nk, a.B * a.Hkv, C::D, C::BN, C::ES))
    return 5;
  FwdParams p;
  p.o_lse = a.lse;
  p.o = (__nv_bfloat16 *)a.o;
  p.Hq = a.Hq; p.Hkv = a.Hkv; p.Nq = a.Nq; p.Nk = a.Nk;
  p.nqb = (a.Nq + C::UROWS - 1) / C::UROWS;
  p.BH = a.B * a.Hq;
  // e4m3: the Q and K descales fold into the score scale
  p.scale_log2 = (float)((double)a.scale * (C::F8 ? (double)a.descale_q * a.descale_k : 1.0) *
                         1.4426950408889634);
  p.causal = a.causal;
  p.causal_off = a.causal_off;
  p.splits = a.splits;
  // Causal order: heaviest query blocks first across all heads.  bf16 d =
  // 256 (one 128-row tile per unit, 128 KB of K and V per key block) with the
  // K/V of all heads above 256 MB: heads go in groups whose K/V fit in 48 MB,
  // so the units in flight re-read K/V from L2 rather than DRAM (measured on
  // B200, causal B4 H16 N8192: 2.24 -> 1.87 ms, B16 N2048 0.80 -> 0.62, B64
  // N512 0.316 -> 0.283; 24 or 96 MB groups were slower; at d = 64 and 128,
  // whose units read a quarter of those bytes per query row, grouping was
  // neutral or slower: causal B4 H16 N4096 d128 0.289 -> 0.326 ms; the
  // dropout instance, bound by its mask warps, gained nothing either way:
  // p = 0.1, B4 H16 N8192 3.04 -> 3.11 ms, B16 N2048 0.97 -> 0.95).
  {
    const double kv_per_head = 2.0 * a.Nk * C::D * C::ES / (double)(a.Hq / a.Hkv);
    const double kv_all = kv_per_head * a.B * a.Hq;
    p.hg = p.BH;
    if (C::D == 256 && C::ES == 2 && !C::MW && a.causal && kv_all > 256.0 * 1024 * 1024) {
      const double hg = (48.0 * 1024 * 1024) / kv_per_head;
      p.hg = hg < 1.0 ? 1 : (hg > p.BH ? p.BH : (int)hg);
    }
  }
  p.o_part = a.splits > 1 ? (float *)a.ws : nullptr;
  p.l_part = a.splits > 1 ? (float *)((char *)a.ws + splitkv_l_offset(a.splits, a.B, a.Hq, a.Nq, a.d))
                          : nullptr;
  p.drop_thr = a.drop_thr;
  p.seed_lo = (uint32_t)a.seed;
  p.seed_hi = (uint32_t)(a.seed >> 32);
  p.drop_off = (uint32_t)a.drop_offset;
  p.o_scale = a.drop_thr != 0 ? a.drop_scale : (C::F8 ? a.descale_v : 1.f);
  p.err = a.err;
  if (a.drop_thr != 0 && a.splits > 1) return 2;   // dropout only in the plain forward
  if (a.drop_thr != 0 && !C::MW) return 2;   // dropout: the mask-warp instances
  if (C::PAIR && a.splits > 1) return 2;      // pairs: plain forward only
  if (C::CSKIP && !(a.causal && a.splits == 1)) return 2;
  auto kern = fwd_kernel<C, C::MW>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
      cudaSuccess)
    return 5;
  const long long units = (long long)p.nqb * p.BH * p.splits;
  if (units > 2147483647LL) return 2;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 5;
  if constexpr (C::PAIR) {
    // clusters of two CTAs, one pair per unit up to the number of pairs
    // that fit at once
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = a.stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3((unsigned)(2 * (sms / 2)), 1, 1);
    int pairs = 0;
    if (cudaOccupancyMaxActiveClusters(&pairs, kern, &cfg) != cudaSuccess || pairs < 1) return 5;
    const long long npairs = units < pairs ? units : pairs;
    cfg.gridDim = dim3((unsigned)(2 * npairs), 1, 1);
    if (cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, p) != cudaSuccess) return 5;
    return cudaGetLastError() == cudaSuccess ? 0 : 5;
  }
  const long long grid = units < sms ? units : sms;
  kern<<<(unsigned)grid, kThreads, C::SMEM, a.stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? 0 : 5;
}

// Merge the pieces of a split-KV forward, one warp per query row:
// L = log sum_s exp(L_s), O = sum_s exp(L_s - L) O_s -> bf16.  The pieces'
// log-sum-exps are reduced across the lanes first; the weighted sum then
// keeps four pieces' loads in flight at a time.
template <int PER>
__device__ __forceinline__ void load_row_slice(const float *src, float (&v)[PER]) {
  if constexpr (PER == 2) {
    const float2 t = *reinterpret_cast<const float2 *>(src);
    v[0] = t.x; v[1] = t.y;
  } else {
#pragma unroll
    for (int e = 0; e < PER; e += 4) {
      const float4 t = *reinterpret_cast<const float4 *>(src + e);
      v[e] = t.x; v[e + 1] = t.y; v[e + 2] = t.z; v[e + 3] = t.w;
    }
  }
}

template <int D>
__global__ void splitkv_combine_kernel(const float *__restrict__ o_part,
                                       const float *__restrict__ l_part, __nv_bfloat16 *__restrict__ o,
                                       float *__restrict__ lse, int splits, long long rows) {
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float *lp = l_part + row;
  float m = -INFINITY;
  for (int s = lane; s < splits; s += 32) m = fmaxf(m, lp[(size_t)s * rows]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float tot = 0.f;
  if (m != -INFINITY) {
    for (int s = lane; s < splits; s += 32) {
      const float ls = lp[(size_t)s * rows];
      tot += ls == -INFINITY ? 0.f : __expf(ls - m);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, off);
  }
  constexpr int PER = D / 32;   // 2, 4 or 8 elements per lane
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  if (tot > 0.f) {
    const float *op = o_part + row * D + lane * PER;
    const size_t piece = (size_t)rows * D;
    int s = 0;
    for (; s + 4 <= splits; s += 4) {
      float w[4], v[4][PER];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float ls = lp[(size_t)(s + u) * rows];
        w[u] = ls == -INFINITY ? 0.f : __expf(ls - m);
        load_row_slice<PER>(op + (size_t)(s + u) * piece, v[u]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] = fmaf(w[u], v[u][e], acc[e]);
    }
    for (; s < splits; ++s) {
      const float ls = lp[(size_t)s * rows];
      const float w = ls == -INFINITY ? 0.f : __expf(ls - m);
      float v[PER];
      load_row_slice<PER>(op + (size_t)s * piece, v);
#pragma unroll
      for (int e = 0; e < PER; ++e) acc[e] = fmaf(w, v[e], acc[e]);
    }
  }
  const float inv = tot > 0.f ? 1.f / tot : 0.f;
  __nv_bfloat16 *dst = o + row * D + lane * PER;
#pragma unroll
  for (int e = 0; e < PER; e += 2)
    *reinterpret_cast<uint32_t *>(dst + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
  if (lane == 0) lse[row] = tot > 0.f ? m + __logf(tot) : -INFINITY;
}

template <int D>
int run_combine(const AttnArgs &a) {
  const long long rows = (long long)a.B * a.Hq * a.Nq;
  const float *o_part = (const float *)a.ws;
  const float *l_part =
      (const float *)((const char *)a.ws + splitkv_l_offset(a.splits, a.B, a.Hq, a.Nq, a.d));
  splitkv_combine_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, a.stream>>>(
      o_part, l_part, (__nv_bfloat16 *)a.o, a.lse, a.splits, rows);
  return cudaGetLastError() == cudaSuccess ? 0 : 5;
}

}  // namespace

int launch_fwd_splitkv_bf16_sm100(const AttnArgs &a) {
  int st = launch_fwd_bf16_sm100(a);
  if (st || a.splits <= 1) return st;
  switch (a.d) {
    case 64: return run_combine<64>(a);
    case 128: return run_combine<128>(a);
    case 256: return run_combine<256>(a);
    default: return 2;
  }
}

// Causal with one piece and at most this many keys: tile 0 stops early (CSKIP).
constexpr int kCskipMaxKeys = 2048;

int launch_fwd_e4m3_sm100(const AttnArgs &a) {
  switch (a.d) {
    case 128:
      return a.causal && a.Nk <= kCskipMaxKeys
                 ? run_fwd<FwdCfg<128, 2, 128, 3, 1, false, false, true>>(a)
                 : run_fwd<FwdCfg<128, 2, 128, 3, 1>>(a);
    case 256: return run_fwd<FwdCfg<256, 1, 128, 2, 1>>(a);
    default: return 2;
  }
}

// CTA-pair forward (bf16, no dropout, plain forward): d = 128 and 256.
int launch_fwd_pair_bf16_sm100(const AttnArgs &a) {
  if (a.drop_thr != 0 || a.splits > 1) return 2;
  switch (a.d) {
    case 128: return run_fwd<FwdCfg<128, 2, 128, 3, 2, false, true>>(a);
    case 256: return run_fwd<FwdCfg<256, 1, 128, 2, 2, false, true>>(a);
    default: return 2;
  }
}

int launch_fwd_bf16_sm100(const AttnArgs &a) {
  switch (a.d) {
    // dropout (not in split mode) at d = 64, 128: one Q tile per CTA, with
    // warps 4-7 evaluating the mask
    // causal, one piece, up to kCskipMaxKeys keys: the instances whose tile 0
    // stops one block early
    case 64:
      if (a.drop_thr && a.splits == 1) return run_fwd<FwdCfg<64, 1, 128, 4, 2, true>>(a);
      if (a.causal && a.splits == 1 && a.Nk <= kCskipMaxKeys)
        return run_fwd<FwdCfg<64, 2, 128, 3, 2, false, false, true>>(a);
      return run_fwd<FwdCfg<64, 2, 128, 3, 2>>(a);
    case 128:
      if (a.drop_thr && a.splits == 1) return run_fwd<FwdCfg<128, 1, 128, 2, 2, true>>(a);
      if (a.causal && a.splits == 1 && a.Nk <= kCskipMaxKeys)
        return run_fwd<FwdCfg<128, 2, 128, 1, 2, false, false, true>>(a);
      return run_fwd<FwdCfg<128, 2, 128, 1, 2>>(a);
    case 256:
      return a.drop_thr && a.splits == 1 ? run_fwd<FwdCfg<256, 1, 128, 1, 2, true>>(a)
                                         : run_fwd<FwdCfg<256, 1, 128, 1, 2>>(a);
    default: return 2;
  }
}

}  // namespace fa
