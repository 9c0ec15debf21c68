// fa_simt.cu -- float32 attention on the CUDA cores (correctness path for
// float32 inputs, where tensor-core TF32 cannot meet a 1e-4 error bound).
//
// Forward: one warp per query row, key/value blocks of 32 rows staged in
// shared memory, the online-softmax recurrence with deferred normalisation
// (FlashAttention blog, section 4.1; CSDN FlashAttention-1 tutorial, section
// 3): running max m, running sum l, unnormalised O rescaled by exp(m_old -
// m_new), one final divide, L = m + ln(l) saved per row.
// Backward: P is recomputed from q, k and L (blog section 2.3); one warp per
// query row accumulates dQ in registers and adds its dK / dV contributions
// with float32 atomics.
#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace fa {
namespace {

constexpr int kRows = 8;    // warps (query rows) per CTA
constexpr int kKeys = 32;   // key rows per block

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Stage key/value rows [j0, j0 + 32) of one head into shared memory with a
// row pitch of d + 1 floats (lane-per-row dot products hit distinct banks).
__device__ __forceinline__ void stage_kv(float *Ks, float *Vs, const float *kh, const float *vh,
                                        int j0, int Nk, int d) {
  const int pitch = d + 1;
  for (int e = threadIdx.x; e < kKeys * d; e += blockDim.x) {
    const int r = e / d, c = e - r * d;
    const int j = j0 + r;
    const bool ok = j < Nk;
    Ks[r * pitch + c] = ok ? kh[(size_t)j * d + c] : 0.f;
    Vs[r * pitch + c] = ok ? vh[(size_t)j * d + c] : 0.f;
  }
}

template <int DPL>
__global__ void __launch_bounds__(kRows * 32) fwd_f32_kernel(const float *__restrict__ q,
                                                             const float *__restrict__ k,
                                                             const float *__restrict__ v,
                                                             float *__restrict__ o,
                                                             float *__restrict__ lse, int Hq,
                                                             int Hkv, int Nq, int Nk, int d,
                                                             float scale, int causal) {
  extern __shared__ float sm[];
  const int pitch = d + 1;
  float *Ks = sm;
  float *Vs = Ks + kKeys * pitch;
  float *Qs = Vs + kKeys * pitch;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (Hq / Hkv);
  const int row = blockIdx.x * kRows + warp;
  const bool active = row < Nq;
  const size_t qbase = ((size_t)b * Hq + h) * Nq;
  const float *kh = k + ((size_t)b * Hkv + kvh) * Nk * d;
  const float *vh = v + ((size_t)b * Hkv + kvh) * Nk * d;

  float *qrow = Qs + warp * d;
  if (active)
    for (int c = lane; c < d; c += 32) qrow[c] = q[(qbase + row) * d + c];

  float acc[DPL];
#pragma unroll
  for (int t = 0; t < DPL; ++t) acc[t] = 0.f;
  float m = -INFINITY, l = 0.f;

  const int key_end = causal ? min(Nk, (int)(blockIdx.x + 1) * kRows) : Nk;
  for (int j0 = 0; j0 < key_end; j0 += kKeys) {
    __syncthreads();
    stage_kv(Ks, Vs, kh, vh, j0, Nk, d);
    __syncthreads();
    if (!active) continue;
    const int j = j0 + lane;
    float s = 0.f;
    const float *krow = Ks + lane * pitch;
    for (int c = 0; c < d; ++c) s = fmaf(qrow[c], krow[c], s);
    s *= scale;
    const bool valid = (j < Nk) && (!causal || j <= row);
    s = valid ? s : -INFINITY;
    const float m_new = fmaxf(m, warp_max(s));
    if (m_new == -INFINITY) continue;  // nothing visible yet
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
    const float p = valid ? expf(s - m_new) : 0.f;
    l = alpha * l + warp_sum(p);
#pragma unroll
    for (int t = 0; t < DPL; ++t) acc[t] *= alpha;
    for (int jj = 0; jj < kKeys; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
      const float *vrow = Vs + jj * pitch;
#pragma unroll
      for (int t = 0; t < DPL; ++t) {
        const int c = lane + 32 * t;
        if (c < d) acc[t] = fmaf(pj, vrow[c], acc[t]);
      }
    }
    m = m_new;
  }
  if (active) {
    const float inv = 1.f / l;
#pragma unroll
    for (int t = 0; t < DPL; ++t) {
      const int c = lane + 32 * t;
      if (c < d) o[(qbase + row) * d + c] = acc[t] * inv;
    }
    if (lane == 0) lse[qbase + row] = m + logf(l);
  }
}

// D_i = sum_c dO_ic * O_ic, one warp per row.
__global__ void bwd_dsum_f32_kernel(const float *__restrict__ o, const float *__restrict__ dout,
                                    float *__restrict__ D, long long rows, int d) {
  const long long row = (long long)blockIdx.x * kRows + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float s = 0.f;
  for (int c = lane; c < d; c += 32) s = fmaf(o[row * d + c], dout[row * d + c], s);
  s = warp_sum(s);
  if (lane == 0) D[row] = s;
}

template <int DPL>
__global__ void __launch_bounds__(kRows * 32) bwd_f32_kernel(
    const float *__restrict__ q, const float *__restrict__ k, const float *__restrict__ v,
    const float *__restrict__ lse, const float *__restrict__ dout, const float *__restrict__ D,
    float *__restrict__ dq, float *__restrict__ dk, float *__restrict__ dv, int Hq, int Hkv,
    int Nq, int Nk, int d, float scale, int causal) {
  extern __shared__ float sm[];
  const int pitch = d + 1;
  float *Ks = sm;
  float *Vs = Ks + kKeys * pitch;
  float *Qs = Vs + kKeys * pitch;
  float *DOs = Qs + kRows * d;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (Hq / Hkv);
  const int row = blockIdx.x * kRows + warp;
  const bool active = row < Nq;
  const size_t qbase = ((size_t)b * Hq + h) * Nq;
  const size_t kvbase = ((size_t)b * Hkv + kvh) * Nk;
  const float *kh = k + kvbase * d;
  const float *vh = v + kvbase * d;

  float *qrow = Qs + warp * d;
  float *dorow = DOs + warp * d;
  float qreg[DPL], doreg[DPL], acc[DPL];
#pragma unroll
  for (int t = 0; t < DPL; ++t) {
    const int c = lane + 32 * t;
    const bool in = active && c < d;
    qreg[t] = in ? q[(qbase + row) * d + c] : 0.f;
    doreg[t] = in ? dout[(qbase + row) * d + c] : 0.f;
    acc[t] = 0.f;
  }
  if (active)
    for (int c = lane; c < d; c += 32) {
      qrow[c] = q[(qbase + row) * d + c];
      dorow[c] = dout[(qbase + row) * d + c];
    }
  const float L = active ? lse[qbase + row] : 0.f;
  const float Di = active ? D[qbase + row] : 0.f;

  const int key_end = causal ? min(Nk, (int)(blockIdx.x + 1) * kRows) : Nk;
  for (int j0 = 0; j0 < key_end; j0 += kKeys) {
    __syncthreads();
    stage_kv(Ks, Vs, kh, vh, j0, Nk, d);
    __syncthreads();
    if (!active) continue;
    const int j = j0 + lane;
    const bool valid = (j < Nk) && (!causal || j <= row);
    float s = 0.f, dp = 0.f;
    const float *krow = Ks + lane * pitch;
    const float *vrow = Vs + lane * pitch;
    for (int c = 0; c < d; ++c) {
      s = fmaf(qrow[c], krow[c], s);
      dp = fmaf(dorow[c], vrow[c], dp);
    }
    const float p = valid ? expf(s * scale - L) : 0.f;
    const float ds = p * (dp - Di);
    for (int jj = 0; jj < kKeys; ++jj) {
      const float dsj = __shfl_sync(0xffffffffu, ds, jj);
      const float pj = __shfl_sync(0xffffffffu, p, jj);
      if (pj == 0.f && dsj == 0.f) continue;  // masked key (warp-uniform)
      const float *kr = Ks + jj * pitch;
      float *dkr = dk + (kvbase + j0 + jj) * d;
      float *dvr = dv + (kvbase + j0 + jj) * d;
#pragma unroll
      for (int t = 0; t < DPL; ++t) {
        const int c = lane + 32 * t;
        if (c < d) {
          acc[t] = fmaf(dsj, kr[c], acc[t]);
          atomicAdd(dkr + c, scale * dsj * qreg[t]);
          atomicAdd(dvr + c, pj * doreg[t]);
        }
      }
    }
  }
  if (active) {
#pragma unroll
    for (int t = 0; t < DPL; ++t) {
      const int c = lane + 32 * t;
      if (c < d) dq[(qbase + row) * d + c] = scale * acc[t];
    }
  }
}

template <typename F>
int dispatch_dpl(int d, F &&f) {
  switch ((d + 31) / 32) {
    case 1: return f(std::integral_constant<int, 1>{});
    case 2: return f(std::integral_constant<int, 2>{});
    case 3: return f(std::integral_constant<int, 3>{});
    case 4: return f(std::integral_constant<int, 4>{});
    case 5: return f(std::integral_constant<int, 5>{});
    case 6: return f(std::integral_constant<int, 6>{});
    case 7: return f(std::integral_constant<int, 7>{});
    case 8: return f(std::integral_constant<int, 8>{});
    default: return 2;
  }
}

}  // namespace

int launch_fwd_f32(const AttnArgs &a) {
  const size_t smem = (size_t)(2 * kKeys * (a.d + 1) + kRows * a.d) * sizeof(float);
  dim3 grid((a.Nq + kRows - 1) / kRows, a.Hq, a.B);
  return dispatch_dpl(a.d, [&](auto dpl) -> int {
    constexpr int DPL = decltype(dpl)::value;
    auto kern = fwd_f32_kernel<DPL>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return 5;
    kern<<<grid, kRows * 32, smem, a.stream>>>(
        (const float *)a.q, (const float *)a.k, (const float *)a.v, (float *)a.o, a.lse, a.Hq,
        a.Hkv, a.Nq, a.Nk, a.d, a.scale, a.causal);
    return cudaGetLastError() == cudaSuccess ? 0 : 5;
  });
}

int launch_bwd_f32(const AttnArgs &a) {
  float *D = (float *)a.ws;
  const long long rows = (long long)a.B * a.Hq * a.Nq;
  const size_t kvbytes = (size_t)a.B * a.Hkv * a.Nk * a.d * sizeof(float);
  if (cudaMemsetAsync(a.dk, 0, kvbytes, a.stream) != cudaSuccess) return 5;
  if (cudaMemsetAsync(a.dv, 0, kvbytes, a.stream) != cudaSuccess) return 5;
  bwd_dsum_f32_kernel<<<(unsigned)((rows + kRows - 1) / kRows), kRows * 32, 0, a.stream>>>(
      (const float *)a.o_in, (const float *)a.dout, D, rows, a.d);
  if (cudaGetLastError() != cudaSuccess) return 5;
  const size_t smem = (size_t)(2 * kKeys * (a.d + 1) + 2 * kRows * a.d) * sizeof(float);
  dim3 grid((a.Nq + kRows - 1) / kRows, a.Hq, a.B);
  return dispatch_dpl(a.d, [&](auto dpl) -> int {
    constexpr int DPL = decltype(dpl)::value;
    auto kern = bwd_f32_kernel<DPL>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return 5;
    kern<<<grid, kRows * 32, smem, a.stream>>>(
        (const float *)a.q, (const float *)a.k, (const float *)a.v, a.lse,
        (const float *)a.dout, D, (float *)a.dq, (float *)a.dk, (float *)a.dv, a.Hq, a.Hkv,
        a.Nq, a.Nk, a.d, a.scale, a.causal);
    return cudaGetLastError() == cudaSuccess ? 0 : 5;
  });
}

}  // namespace fa
