// launch.h -- internal host-side launchers behind the C ABI (not exported).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

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
  cudaStream_t stream = nullptr;
  unsigned *err = nullptr;      // device error word
};

// Byte offset of the dQ accumulator inside the workspace.
inline size_t ws_dq_offset(int B, int Hq, int Nq) {
  size_t dbytes = (size_t)B * Hq * Nq * sizeof(float);
  return (dbytes + 255) & ~(size_t)255;
}

// Status codes use the fa_status numbering of fa.h.
int launch_fwd_f32(const AttnArgs &a);
int launch_bwd_f32(const AttnArgs &a);
int launch_fwd_bf16_sm100(const AttnArgs &a);
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
