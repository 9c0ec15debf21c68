// launch.h -- internal host-side launchers behind the C ABI (not exported).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

struct AttnArgs {
  const void *q = nullptr, *k = nullptr, *v = nullptr;
  const void *o_in = nullptr;   // forward output (backward input)
  const void *dout = nullptr;
  void *o = nullptr;            // forward output
  float *lse = nullptr;         // forward output / backward input
  void *dq = nullptr, *dk = nullptr, *dv = nullptr;
  void *ws = nullptr;           // backward workspace: D then dQ accumulator
  int B = 0, Hq = 0, Hkv = 0, Nq = 0, Nk = 0, d = 0;
  float scale = 0.f;
  int causal = 0;
  int causal_off = 0;           // causal: key j hidden from query i when j > i + causal_off
  int splits = 1;               // split-KV forward: pieces of the key range (ws holds them)
  // dropout on P: keep element (b, h, i, j) when word j % 4 of
  // Philox4x32-10(key = seed, counter = (j / 4, i, b*Hq + h, offset)) is
  // >= drop_thr = floor(p * 2^32); 0 = no dropout.  drop_scale = 1 / (1 - p).
  uint32_t drop_thr = 0;
  float drop_scale = 1.f;
  unsigned long long seed = 0, drop_offset = 0;
  // e4m3 forward: per-tensor dequantisation factors (tensor = factor * code value)
  float descale_q = 1.f, descale_k = 1.f, descale_v = 1.f;
  cudaStream_t stream = nullptr;
  unsigned *err = nullptr;      // device error word
};

// Backward workspace layout (float32 throughout, offsets in bytes):
//   D   [B*Hq][Npad]   rowsum(dO * O); rows past Nq hold 0
//   L2  [B*Hq][Npad]   log2e * L - scale*log2e * (q . c): the log-sum-exp in
//                      base 2, shifted for the centred K; rows past Nq +inf
//   c   [B*Hq][d]      per key/value head centring vector (first B*Hkv*d used)
//   n   int32          work counter of the persistent dK/dV kernel (zeroed by prep)
//   dQ  [B*Hq][Nq][d]  dQ accumulator, 256-byte aligned
// Npad = Nq rounded up to 128, so every 64- or 128-row query block of D and
// L2 is a 256-byte aligned block a bulk copy can fetch.
inline size_t ws_npad(int Nq) { return (size_t)((Nq + 127) / 128) * 128; }
inline size_t ws_l2_offset(int B, int Hq, int Nq) { return (size_t)B * Hq * ws_npad(Nq) * 4; }
inline size_t ws_c_offset(int B, int Hq, int Nq) { return 2 * ws_l2_offset(B, Hq, Nq); }
inline size_t ws_sched_offset(int B, int Hq, int Nq, int d) {
  return ws_c_offset(B, Hq, Nq) + (size_t)B * Hq * d * 4;
}
inline size_t ws_dq_offset(int B, int Hq, int Nq, int d) {
  return (ws_sched_offset(B, Hq, Nq, d) + 16 + 255) & ~(size_t)255;
}
inline size_t ws_bytes(int B, int Hq, int Nq, int d) {
  return ws_dq_offset(B, Hq, Nq, d) + (size_t)B * Hq * Nq * d * 4;
}

// Split-KV forward workspace (float32): normalised partial outputs
// [splits][B*Hq][Nq][d], then (256-byte aligned) partial log-sum-exps
// [splits][B*Hq][Nq].
inline size_t splitkv_l_offset(int splits, int B, int Hq, int Nq, int d) {
  return ((size_t)splits * B * Hq * Nq * d * 4 + 255) & ~(size_t)255;
}
inline size_t splitkv_ws_bytes(int splits, int B, int Hq, int Nq, int d) {
  return splitkv_l_offset(splits, B, Hq, Nq, d) + (size_t)splits * B * Hq * Nq * 4;
}

// Status codes use the fa_status numbering of fa.h.
int launch_fwd_f32(const AttnArgs &a);
int launch_bwd_f32(const AttnArgs &a);
int launch_fwd_bf16_sm100(const AttnArgs &a);
int launch_fwd_splitkv_bf16_sm100(const AttnArgs &a);   // pieces + merge (splits > 1)
int launch_fwd_pair_bf16_sm100(const AttnArgs &a);      // CTA-pair form (d = 128, 256)
int launch_fwd_e4m3_sm100(const AttnArgs &a);   // e4m3 Q/K/V, bf16 O (d = 128, 256)
int launch_bwd_bf16_sm100(const AttnArgs &a);   // all three stages
int launch_bwd_prep_bf16(const AttnArgs &a);     // D + zeroed dQ accumulator
int launch_bwd_dkdv_bf16_sm100(const AttnArgs &a);
int launch_bwd_dq_bf16(const AttnArgs &a);       // dq = bf16(scale * accumulator)
int launch_wait_selftest(long long timeout_ns, cudaStream_t stream, unsigned *err);

// Argument checks and per-call device set-up shared by the C entry points
// (fa_status codes): size/scale rules, then current device, architecture and
// the device error word.
int validate_sizes(int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal);
int device_prologue(int *dev, AttnArgs &a);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_tiled();

}  // namespace fa
