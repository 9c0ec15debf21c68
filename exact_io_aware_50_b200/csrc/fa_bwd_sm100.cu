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
// Three launches on the caller's stream:
//   1. preprocess: D_i = sum_d dO_id O_id (f32) and a zeroed f32 dQ
//      accumulator, both in the caller's workspace;
//   2. the dK/dV kernel: one CTA per (batch, key/value head, 128-row key
//      block); it keeps K_j, V_j in shared memory and dK_j, dV_j in TMEM
//      for the whole loop over the query heads of its group and their 64-row
//      query blocks, so dK and dV need no atomics.  Per step (transposed
//      forms, key rows on the 128 TMEM lanes):
//          S^T  = K_j Q_i^T          dP^T = V_j dO_i^T     (tcgen05, SMEM x SMEM)
//          P^T  = exp2(S^T * scale*log2e - L_i*log2e),  dS^T = P^T * (dP^T - D_i)
//                                                          (one thread per key row)
//          dV  += P^T dO_i           dK  += dS^T Q_i       (tcgen05, A from TMEM)
//          dQ_i^T = K_j^T dS^T                             (tcgen05, SMEM x SMEM)
//      and a readout warpgroup adds dQ_i^T into the f32 accumulator with
//      float32 reductions.  Two TMEM sets (S^T|dP^T, reused for P^T|dS^T and
//      dQ^T) let S^T/dP^T of step i+1 run while step i is in the elementwise
//      stage;
//   3. convert: dQ = bf16(scale * accumulator).
#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace fa {
namespace {

constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kCenterRows = 64;   // rows of K averaged into the centering vector c

// Pass layouts.  kFull: dK, dV and dQ in one pass (d = 64, 128).  For
// d = 256 the dK and dV accumulators alone fill TMEM, so the work is split
// into two launches over the same key blocks: kDV (S^T, P^T, dV) and kDKDQ
// (S^T, dP^T, dS^T, dK, dQ).
enum Mode { kFull = 0, kDV = 1, kDKDQ = 2 };

template <int D_, int MODE_>
struct BwdCfg {
  static constexpr int D = D_, MODE = MODE_;
  static constexpr int BN = 128;       // key rows per CTA (MMA M)
  static constexpr int BM = 64;        // query rows per step (MMA N)
  static constexpr int NSETS = MODE == kDKDQ ? 1 : 2;   // TMEM score sets
  static constexpr int QS = MODE == kDKDQ ? 1 : 2;      // query-stage ring depth
  static constexpr bool HAS_DP = MODE != kDV;
  static constexpr bool HAS_DV = MODE != kDKDQ;
  static constexpr bool HAS_DK = MODE != kDV;
  static constexpr bool HAS_DQ = MODE != kDV;
  // dQ uses K - c (c: per-head constant vector); see the kernel comment.
  static constexpr bool CENTER = MODE == kFull;
  static constexpr int DCH = D / 64;   // 128-byte column chunks
  static constexpr int KV_CHUNK = BN * 128;
  static constexpr int KV_TILE = KV_CHUNK * DCH;
  static constexpr int Q_CHUNK = BM * 128;
  static constexpr int Q_TILE = Q_CHUNK * DCH;
  static constexpr int DS_TILE = BN * BM * 2;  // dS^T, bf16, one 128-byte chunk wide
  static_assert(BM == 64, "dS^T buffer is one 64-element swizzle chunk wide");
  static constexpr int OFF_K = 0;
  static constexpr int OFF_KC = OFF_K + KV_TILE;                       // centred K (CENTER)
  static constexpr int OFF_V = OFF_KC + (CENTER ? KV_TILE : 0);         // V (HAS_DP); follows KC
  static constexpr int OFF_Q = OFF_V + (HAS_DP ? KV_TILE : 0);
  static constexpr int OFF_DO = OFF_Q + QS * Q_TILE;
  static constexpr int OFF_DS = OFF_DO + QS * Q_TILE;
  static constexpr int OFF_LSE = OFF_DS + (HAS_DQ ? NSETS * DS_TILE : 0);  // QS x BM floats
  static constexpr int OFF_DD = OFF_LSE + QS * BM * 4;                      // QS x BM floats
  static constexpr int OFF_C = OFF_DD + QS * BM * 4;                        // D floats
  static constexpr int OFF_BAR = OFF_C + D * 4;
  // kv_full, kc_full, q_full[QS], q_empty[QS], s_full[2], p_full[2],
  // dq_full[2], dq_empty[2], final, drain
  static constexpr int NBAR = 2 + 2 * QS + 8 + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  // TMEM columns.
  //   kFull : dV [0, D), dK [D, 2D), set x at 2D + 128x:
  //           S^T [0,64) dP^T [64,128); then P^T [0,32) dS^T [32,64) dQ^T [64,128)
  //   kDV   : dV [0, 256), set x at 256 + 64x: S^T [0,64); then P^T [0,32)
  //   kDKDQ : dK [0, 256), set at 256: S^T [0,64) dP^T [64,128);
  //           then dS^T [32,64), dQ^T halves [128,192) and [192,256)
  static constexpr int TM_DV = 0;
  static constexpr int TM_DK = MODE == kFull ? D : 0;
  static constexpr int TM_SET0 = MODE == kFull ? 2 * D : D;
  static constexpr int SET_STRIDE = MODE == kDV ? 64 : 128;
  static constexpr int TM_DQ = MODE == kFull ? 64 : 128;   // dQ^T offset inside its set
  static constexpr int TM_ALLOC = 512;
  static_assert(TM_SET0 + NSETS * SET_STRIDE + (MODE == kDKDQ ? 128 : 0) <= TM_ALLOC, "TMEM");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(MODE != kFull || D <= 128, "full pass needs d <= 128");
  static_assert(MODE == kFull || D == 256, "split passes are for d = 256");
};

struct BwdParams {
  const float *lse;        // [B, Hq, Nq]
  const float *Dsum;       // [B, Hq, Nq]
  float *dq_acc;           // [B, Hq, Nq, D]
  const __nv_bfloat16 *k;  // [B, Hkv, Nk, D] (for the centering vector)
  __nv_bfloat16 *dk, *dv;  // [B, Hkv, Nk, D]
  int Hq, Hkv, Nq, Nk, nqb, nkb, BHkv;
  float scale, scale_log2;
  int causal;
  unsigned *err;
};

// dQ and the mean of K.  Every row of dS sums to zero (sum_j P_ij dP_ij =
// D_i and sum_j P_ij = 1), so dQ_i = scale * sum_j dS_ij (k_j - c) for any
// vector c that is the same for all key rows of the head.  With c near the
// mean of K, the bf16 rounding of dS is no longer multiplied by the mean of
// K (the +8-shifted K workload makes that term 8x the rest).  c is the f32
// mean of the head's first min(Nk, 64) key rows, computed identically by
// every CTA of the head.
template <class C>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
               const BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t *bars = (uint64_t *)(smem + C::OFF_BAR);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const int B_KV = 0, B_KC = 1, B_QFULL = 2, B_QEMPTY = 2 + C::QS, B_SFULL = 2 + 2 * C::QS,
            B_PFULL = B_SFULL + 2, B_DQFULL = B_PFULL + 2, B_DQEMPTY = B_DQFULL + 2,
            B_FINAL = B_DQEMPTY + 2, B_DRAIN = B_FINAL + 1;
  uint32_t *tmem_slot = (uint32_t *)(smem + C::OFF_MISC);
  volatile int *abort_flag = (volatile int *)(smem + C::OFF_MISC + 4);
  float *s_lse = (float *)(smem + C::OFF_LSE);
  float *s_dd = (float *)(smem + C::OFF_DD);
  float *s_c = (float *)(smem + C::OFF_C);

  const int warp = warp_id_uniform();
  const int lane = threadIdx.x & 31;

  // Work unit: key blocks with the most query blocks first (causal), then
  // (batch, key/value head).
  const int unit = blockIdx.x;
  const int jblk = unit / p.BHkv;
  const int bhkv = unit % p.BHkv;
  const int b = bhkv / p.Hkv, hkv = bhkv % p.Hkv;
  const int g = p.Hq / p.Hkv;
  const int kv0 = jblk * C::BN;
  const int i0 = p.causal ? kv0 / C::BM : 0;  // first query block that sees this key block
  const int nq_eff = p.nqb - i0;
  const int nsteps = nq_eff > 0 ? g * nq_eff : 0;
  auto step_head = [&](int s) { return hkv * g + s / nq_eff; };
  auto step_qblk = [&](int s) { return i0 + s % nq_eff; };
  auto set_of = [&](int s) { return C::NSETS == 2 ? (s & 1) : 0; };
  auto set_phase = [&](int s) { return (uint32_t)((C::NSETS == 2 ? (s >> 1) : s) & 1); };

  if (threadIdx.x == 0) {
    mbar_init(bar(B_KV), 1);
    mbar_init(bar(B_KC), 128);
    for (int s = 0; s < C::QS; ++s) {
      mbar_init(bar(B_QFULL + s), 1);
      mbar_init(bar(B_QEMPTY + s), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(B_SFULL + x), 1);
      mbar_init(bar(B_PFULL + x), 128);
      mbar_init(bar(B_DQFULL + x), 1);
      mbar_init(bar(B_DQEMPTY + x), 128);
    }
    mbar_init(bar(B_FINAL), 1);
    mbar_init(bar(B_DRAIN), 1);
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
    int last_phase[C::QS];
    for (int s = 0; s < C::QS; ++s) last_phase[s] = -1;
    bool ok = true;
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(B_KV), (C::HAS_DP ? 2 : 1) * C::KV_TILE);
      for (int c = 0; c < C::DCH; ++c) {
        tma_load_3d(sbase + C::OFF_K + c * C::KV_CHUNK, &tmK, bar(B_KV), c * 64, kv0, bhkv);
        if (C::HAS_DP)
          tma_load_3d(sbase + C::OFF_V + c * C::KV_CHUNK, &tmV, bar(B_KV), c * 64, kv0, bhkv);
      }
    }
    for (int i = 0; i < nsteps && ok; ++i) {
      const int st = i % C::QS;
      const uint32_t ph = (i / C::QS) & 1;
      ok = warp_wait_one(bar(B_QEMPTY + st), ph ^ 1, wc);
      if (!ok) break;
      const int h = step_head(i), qb = step_qblk(i);
      const int bh = b * p.Hq + h;
      const size_t rowbase = (size_t)bh * p.Nq;
      for (int c = lane; c < C::BM; c += 32) {
        const int q = qb * C::BM + c;
        const bool in = q < p.Nq;
        s_lse[st * C::BM + c] = in ? p.lse[rowbase + q] * kLog2e : INFINITY;
        s_dd[st * C::BM + c] = in ? p.Dsum[rowbase + q] : 0.f;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(bar(B_QFULL + st), 2 * C::Q_TILE);
        for (int c = 0; c < C::DCH; ++c) {
          tma_load_3d(sbase + C::OFF_Q + st * C::Q_TILE + c * C::Q_CHUNK, &tmQ, bar(B_QFULL + st),
                      c * 64, qb * C::BM, bh);
          tma_load_3d(sbase + C::OFF_DO + st * C::Q_TILE + c * C::Q_CHUNK, &tmDO,
                      bar(B_QFULL + st), c * 64, qb * C::BM, bh);
        }
      }
      last_phase[st] = ph;
    }
    if (!ok && lane == 0) {
      (void)drain_wait(bar(B_KV), 0, p.err, kWaitLimitNs);
      for (int s = 0; s < C::QS; ++s)
        if (last_phase[s] >= 0) (void)drain_wait(bar(B_QFULL + s), last_phase[s], p.err, kWaitLimitNs);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t IDESC_SP = idesc_bf16(128, C::BM, 0, 0);  // S^T, dP^T: K-major A and B
    constexpr uint32_t IDESC_KV = idesc_bf16(128, C::D, 0, 1);   // dV, dK: A TMEM, B MN-major
    constexpr uint32_t IDESC_DQ = idesc_bf16(128, C::BM, 1, 1);  // dQ^T: both MN-major
    auto issue_SdP = [&](int x, int st) {
      const uint32_t qa = sbase + C::OFF_Q + st * C::Q_TILE;
      const uint32_t da = sbase + C::OFF_DO + st * C::Q_TILE;
      const uint32_t set = tmem + C::TM_SET0 + x * C::SET_STRIDE;
#pragma unroll
      for (int kk = 0; kk < C::D / 16; ++kk) {
        const uint32_t okv = (kk >> 2) * C::KV_CHUNK + (kk & 3) * 32;
        const uint32_t oq = (kk >> 2) * C::Q_CHUNK + (kk & 3) * 32;
        mma_ss(set, sw128_desc(sbase + C::OFF_K + okv, 16, 1024), sw128_desc(qa + oq, 16, 1024),
               IDESC_SP, kk > 0);
      }
      if (C::HAS_DP) {
#pragma unroll
        for (int kk = 0; kk < C::D / 16; ++kk) {
          const uint32_t okv = (kk >> 2) * C::KV_CHUNK + (kk & 3) * 32;
          const uint32_t oq = (kk >> 2) * C::Q_CHUNK + (kk & 3) * 32;
          mma_ss(set + 64, sw128_desc(sbase + C::OFF_V + okv, 16, 1024),
                 sw128_desc(da + oq, 16, 1024), IDESC_SP, kk > 0);
        }
      }
    };
    // dV += P^T dO_i and dK += dS^T Q_i (K = 64 query rows, 16 per MMA)
    auto issue_dvdk = [&](int x, int st, bool first) {
      const uint32_t qa = sbase + C::OFF_Q + st * C::Q_TILE;
      const uint32_t da = sbase + C::OFF_DO + st * C::Q_TILE;
      const uint32_t set = tmem + C::TM_SET0 + x * C::SET_STRIDE;
      if (C::HAS_DV) {
#pragma unroll
        for (int kk = 0; kk < C::BM / 16; ++kk)
          mma_ts(tmem + C::TM_DV, set + kk * 8, sw128_desc(da + kk * 2048, C::Q_CHUNK, 1024),
                 IDESC_KV, (!first) || kk > 0);
      }
      if (C::HAS_DK) {
#pragma unroll
        for (int kk = 0; kk < C::BM / 16; ++kk)
          mma_ts(tmem + C::TM_DK, set + 32 + kk * 8, sw128_desc(qa + kk * 2048, C::Q_CHUNK, 1024),
                 IDESC_KV, (!first) || kk > 0);
      }
    };
    // dQ_i^T = A^T dS^T with K = 128 key rows (16 per MMA) and M = 128 rows of
    // A^T: [Kc^T ; V^T] for d = 64 (the V half is unused), Kc^T for d = 128,
    // and the two 128-row halves of K^T for d = 256.
    auto issue_dq = [&](int x) {
      const uint32_t set = tmem + C::TM_SET0 + x * C::SET_STRIDE;
      const uint32_t dsb = sbase + C::OFF_DS + x * C::DS_TILE;
      const uint32_t abase = sbase + (C::CENTER ? C::OFF_KC : C::OFF_K);
#pragma unroll
      for (int half = 0; half < (C::D == 256 ? 2 : 1); ++half) {
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk)
          mma_ss(set + C::TM_DQ + half * 64,
                 sw128_desc(abase + half * 2 * C::KV_CHUNK + kk * 2048, C::KV_CHUNK, 1024),
                 sw128_desc(dsb + kk * 2048, C::DS_TILE, 1024), IDESC_DQ, kk > 0);
      }
    };
    bool ok = warp_wait_one(bar(B_KV), 0, wc);
    if (ok && nsteps > 0) {
      ok = warp_wait_one(bar(B_QFULL + 0), 0, wc);
      if (ok) {
        tc_fence_after();
        if (lane == 0) {
          issue_SdP(0, 0);
          mma_commit(bar(B_SFULL + 0));
        }
        __syncwarp();
      }
    }
    if (ok && C::CENTER && nsteps > 0) ok = warp_wait_one(bar(B_KC), 0, wc);
    for (int i = 0; i < nsteps && ok; ++i) {
      const int x = set_of(i);
      const int st = i % C::QS;
      if (C::NSETS == 2 && i + 1 < nsteps) {
        const int y = x ^ 1;
        if (C::HAS_DQ && i >= 1) {
          ok = warp_wait_one(bar(B_DQEMPTY + y), set_phase(i - 1), wc);
          if (!ok) break;
        }
        const int st1 = (i + 1) % C::QS;
        ok = warp_wait_one(bar(B_QFULL + st1), ((i + 1) / C::QS) & 1, wc);
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          issue_SdP(y, st1);
          mma_commit(bar(B_SFULL + y));
        }
        __syncwarp();
      }
      ok = warp_wait_one(bar(B_PFULL + x), set_phase(i), wc);
      if (!ok) break;
      if (C::HAS_DQ && C::NSETS == 1 && i >= 1) {
        ok = warp_wait_one(bar(B_DQEMPTY + x), set_phase(i - 1), wc);
        if (!ok) break;
      }
      tc_fence_after();
      if (lane == 0) {
        issue_dvdk(x, st, i == 0);
        if (C::HAS_DQ) {
          issue_dq(x);
          mma_commit(bar(B_DQFULL + x));
        }
        mma_commit(bar(B_QEMPTY + st));
      }
      __syncwarp();
      if (C::NSETS == 1 && i + 1 < nsteps) {
        const int st1 = (i + 1) % C::QS;
        ok = warp_wait_one(bar(B_QFULL + st1), ((i + 1) / C::QS) & 1, wc);
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          issue_SdP(x, st1);
          mma_commit(bar(B_SFULL + x));
        }
        __syncwarp();
      }
    }
    if (ok) {
      if (lane == 0) mma_commit(bar(B_FINAL));
      __syncwarp();
    } else {
      if (lane == 0) {
        mma_commit(bar(B_DRAIN));
        (void)drain_wait(bar(B_DRAIN), 0, p.err, kWaitLimitNs);
      }
      __syncwarp();
    }
  } else if (warp < 4) {
    // ------------------------------------------------ elementwise stage
    const int r = threadIdx.x;                     // key row within the block = TMEM lane
    const int kv = kv0 + r;
    const bool kv_live = kv < p.Nk;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    bool ok = true;
    if (C::CENTER) {
      // c = mean of the head's first rows of K (f32, fixed order)
      if (r < C::D) {
        const __nv_bfloat16 *kh = p.k + (size_t)bhkv * p.Nk * C::D + r;
        const int nr = min(p.Nk, kCenterRows);
        float acc = 0.f;
        for (int j = 0; j < nr; ++j) acc += __bfloat162float(kh[(size_t)j * C::D]);
        s_c[r] = acc / (float)nr;
      }
      named_barrier_sync(1, 128);
      ok = warp_wait_all(bar(B_KV), 0, wc);
      if (ok) {
        // Kc row r = bf16(K row r - c) in the same swizzled layout (zero past Nk)
#pragma unroll 1
        for (int ch = 0; ch < C::DCH; ++ch) {
          const uint8_t *src = smem + C::OFF_K + ch * C::KV_CHUNK + r * 128;
          uint8_t *dst = smem + C::OFF_KC + ch * C::KV_CHUNK + r * 128;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int col = ch * 64 + ((u ^ (r & 7)) << 3);
            uint4 v = *reinterpret_cast<const uint4 *>(src + (u << 4));
            uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 h2 = *reinterpret_cast<__nv_bfloat162 *>(&w[e]);
              const float2 f = __bfloat1622float2(h2);
              w[e] = kv_live ? pack_bf16x2(f.x - s_c[col + 2 * e], f.y - s_c[col + 2 * e + 1]) : 0u;
            }
            *reinterpret_cast<uint4 *>(dst + (u << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(bar(B_KC));
      }
    }
    for (int i = 0; i < nsteps && ok; ++i) {
      const int x = set_of(i), st = i % C::QS;
      ok = warp_wait_all(bar(B_QFULL + st), (i / C::QS) & 1, wc);
      if (ok) ok = warp_wait_all(bar(B_SFULL + x), set_phase(i), wc);
      if (!ok) break;
      tc_fence_after();
      const uint32_t set = tmem + lane_off + C::TM_SET0 + x * C::SET_STRIDE;
      uint32_t sv[64], dv[64];
      tmem_ld32(set, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld32(set + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      if (C::HAS_DP) {
        tmem_ld32(set + 64, *reinterpret_cast<uint32_t(*)[32]>(&dv[0]));
        tmem_ld32(set + 96, *reinterpret_cast<uint32_t(*)[32]>(&dv[32]));
      }
      tmem_wait_ld();
      const float *lse2 = s_lse + st * C::BM;
      const float *dd = s_dd + st * C::BM;
      const int q0 = step_qblk(i) * C::BM;
      // causal: key kv is hidden from query q when kv > q; key rows past Nk
      // (zero-filled) are masked so they add nothing anywhere
      const int first_vis = !kv_live ? C::BM : (p.causal ? kv - q0 : 0);
      uint32_t pk[32], dk[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        float pr[2], ds[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int c = 2 * e + u;
          float pv = fast_exp2(fmaf(__uint_as_float(sv[c]), p.scale_log2, -lse2[c]));
          pv = (c >= first_vis) ? pv : 0.f;
          pr[u] = pv;
          ds[u] = C::HAS_DP ? pv * (__uint_as_float(dv[c]) - dd[c]) : 0.f;
        }
        pk[e] = pack_bf16x2(pr[0], pr[1]);
        dk[e] = pack_bf16x2(ds[0], ds[1]);
      }
      if (C::HAS_DV) tmem_st32(set, pk);
      if (C::HAS_DK) tmem_st32(set + 32, dk);
      if (C::HAS_DQ) {
        // dS^T row r -> shared memory (B operand of the dQ^T MMA, 128-byte
        // swizzled rows: 16-byte chunk c of row r sits at chunk c ^ (r % 8))
        uint8_t *dsrow = smem + C::OFF_DS + x * C::DS_TILE + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4 *>(dsrow + ((c ^ (r & 7)) << 4)) =
              make_uint4(dk[4 * c], dk[4 * c + 1], dk[4 * c + 2], dk[4 * c + 3]);
        fence_proxy_async_smem();
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_PFULL + x));
    }
    // ------------------------------------------------------ epilogue
    if (ok) ok = warp_wait_all(bar(B_FINAL), 0, wc);
    if (ok && nsteps > 0) {
      tc_fence_after();
      const size_t rowoff = ((size_t)bhkv * p.Nk + (kv_live ? kv : 0)) * C::D;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        if (which == 0 && !C::HAS_DV) continue;
        if (which == 1 && !C::HAS_DK) continue;
        const uint32_t src = tmem + lane_off + (which ? C::TM_DK : C::TM_DV);
        __nv_bfloat16 *dst = (which ? p.dk : p.dv) + rowoff;
        const float mul = which ? p.scale : 1.f;
#pragma unroll 1
        for (int c = 0; c < C::D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(src + c * 32, v);
          tmem_wait_ld();
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
    } else if (ok && nsteps == 0 && kv_live) {
      // no query row sees this key block: its gradients are zero
      const size_t rowoff = ((size_t)bhkv * p.Nk + kv) * C::D;
      for (int e = 0; e < C::D / 8; ++e) {
        if (C::HAS_DK) reinterpret_cast<uint4 *>(p.dk + rowoff)[e] = make_uint4(0, 0, 0, 0);
        if (C::HAS_DV) reinterpret_cast<uint4 *>(p.dv + rowoff)[e] = make_uint4(0, 0, 0, 0);
      }
    }
  } else if (warp < 8 && C::HAS_DQ) {
    // ------------------------------------------------ dQ readout
    const int t = threadIdx.x - 128;               // TMEM lane = column d of dQ (per half)
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    for (int i = 0; i < nsteps; ++i) {
      const int x = set_of(i);
      if (!warp_wait_all(bar(B_DQFULL + x), set_phase(i), wc)) break;
      tc_fence_after();
      const int h = step_head(i), q0 = step_qblk(i) * C::BM;
      const int nvalid = min(C::BM, p.Nq - q0);
      float *acc = p.dq_acc + (((size_t)(b * p.Hq + h)) * p.Nq + q0) * C::D + t;
      constexpr int NH = C::D == 256 ? 2 : 1;
#pragma unroll 1
      for (int half = 0; half < NH; ++half) {
        uint32_t v[64];
        const uint32_t src = tmem + lane_off + C::TM_SET0 + x * C::SET_STRIDE + C::TM_DQ + half * 64;
        tmem_ld32(src, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld32(src + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_wait_ld();
        if (half == NH - 1) {
          tc_fence_before();
          mbar_arrive(bar(B_DQEMPTY + x));
        }
        if (t < C::D) {
          float *a = acc + half * 128;
#pragma unroll
          for (int c = 0; c < C::BM; ++c)
            if (c < nvalid) atomicAdd(a + (size_t)c * C::D, __uint_as_float(v[c]));
        }
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

// D_i = sum_d dO_id * O_id in f32 (one warp per row) and zero the dQ
// accumulator rows of this warp.
template <int D>
__global__ void bwd_preprocess_kernel(const __nv_bfloat16 *__restrict__ o,
                                      const __nv_bfloat16 *__restrict__ dout,
                                      float *__restrict__ Dsum, float *__restrict__ dq_acc,
                                      long long rows) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  constexpr int PER = D / 32;  // elements per lane (2, 4 or 8)
  float s = 0.f;
  const __nv_bfloat16 *orow = o + row * D + lane * PER;
  const __nv_bfloat16 *drow = dout + row * D + lane * PER;
#pragma unroll
  for (int e = 0; e < PER; e += 2) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(orow + e));
    const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(drow + e));
    s = fmaf(a.x, c.x, s);
    s = fmaf(a.y, c.y, s);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) Dsum[row] = s;
  float4 *z = reinterpret_cast<float4 *>(dq_acc + row * D);
  for (int e = lane; e < D / 4; e += 32) z[e] = make_float4(0.f, 0.f, 0.f, 0.f);
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

template <int D>
int run_prep(const AttnArgs &a) {
  float *Dsum = (float *)a.ws;
  float *dq_acc = (float *)((char *)a.ws + ws_dq_offset(a.B, a.Hq, a.Nq));
  const long long rows = (long long)a.B * a.Hq * a.Nq;
  bwd_preprocess_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, a.stream>>>(
      (const __nv_bfloat16 *)a.o_in, (const __nv_bfloat16 *)a.dout, Dsum, dq_acc, rows);
  return cudaGetLastError() == cudaSuccess ? 0 : 5;
}

template <class C>
int run_dkdv(const AttnArgs &a) {
  float *Dsum = (float *)a.ws;
  float *dq_acc = (float *)((char *)a.ws + ws_dq_offset(a.B, a.Hq, a.Nq));
  CUtensorMap mq, mk, mv, mdo;
  if (!make_map(&mq, a.q, a.Nq, a.B * a.Hq, C::D, C::BM) ||
      !make_map(&mdo, a.dout, a.Nq, a.B * a.Hq, C::D, C::BM) ||
      !make_map(&mk, a.k, a.Nk, a.B * a.Hkv, C::D, C::BN) ||
      !make_map(&mv, a.v, a.Nk, a.B * a.Hkv, C::D, C::BN))
    return 5;
  BwdParams p;
  p.lse = a.lse;
  p.k = (const __nv_bfloat16 *)a.k;
  p.Dsum = Dsum;
  p.dq_acc = dq_acc;
  p.dk = (__nv_bfloat16 *)a.dk;
  p.dv = (__nv_bfloat16 *)a.dv;
  p.Hq = a.Hq; p.Hkv = a.Hkv; p.Nq = a.Nq; p.Nk = a.Nk;
  p.nqb = (a.Nq + C::BM - 1) / C::BM;
  p.nkb = (a.Nk + C::BN - 1) / C::BN;
  p.BHkv = a.B * a.Hkv;
  p.scale = a.scale;
  p.scale_log2 = a.scale * kLog2e;
  p.causal = a.causal;
  p.err = a.err;
  auto kern = bwd_kernel<C>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
      cudaSuccess)
    return 5;
  const long long units = (long long)p.nkb * p.BHkv;
  if (units > 2147483647LL) return 2;
  kern<<<(unsigned)units, kThreads, C::SMEM, a.stream>>>(mq, mk, mv, mdo, p);
  return cudaGetLastError() == cudaSuccess ? 0 : 5;
}

int run_dq(const AttnArgs &a) {
  const float *dq_acc = (const float *)((const char *)a.ws + ws_dq_offset(a.B, a.Hq, a.Nq));
  const long long n8 = (long long)a.B * a.Hq * a.Nq * a.d / 8;
  bwd_convert_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, a.stream>>>(
      dq_acc, (__nv_bfloat16 *)a.dq, n8, a.scale);
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

int launch_bwd_dkdv_bf16_sm100(const AttnArgs &a) {
  switch (a.d) {
    case 64: return run_dkdv<BwdCfg<64, kFull>>(a);
    case 128: return run_dkdv<BwdCfg<128, kFull>>(a);
    case 256: {
      int st = run_dkdv<BwdCfg<256, kDV>>(a);
      return st ? st : run_dkdv<BwdCfg<256, kDKDQ>>(a);
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
