// fa_capi.cu -- the C ABI declared in include/fa.h: argument checks, the
// device error word, and dispatch to the kernels' launchers.
#include <math.h>
#include <stdint.h>

#include "../../include/fa.h"
#include "common.cuh"
#include "launch.h"

namespace fa {

// Library device error word (one per device that loads the library).  Bits
// are ErrorBits; fa_device_status() reads and clears it.
__device__ unsigned g_error_word = 0;

namespace {

constexpr int kMaxDevices = 64;
unsigned *g_err_ptr[kMaxDevices] = {};

int current_device_checked(int *dev) {
  if (cudaGetDevice(dev) != cudaSuccess) return FA_ERR_CUDA;
  if (*dev < 0 || *dev >= kMaxDevices) return FA_ERR_CUDA;
  return FA_OK;
}

// Device address of the error word on the current device (looked up once).
unsigned *error_word(int dev) {
  if (!g_err_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = (unsigned *)p;
  }
  return g_err_ptr[dev];
}

int check_arch(int dev) {
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return FA_ERR_CUDA;
  return (major == 10 && minor == 0) ? FA_OK : FA_ERR_ARCH;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// bottom_right: causal with Nq <= Nk allowed (split-KV forward); otherwise
// causal requires Nq == Nk.
int check_sizes(int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                bool bottom_right = false) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Nq <= 0 || Nk <= 0 || d <= 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (causal && (bottom_right ? Nq > Nk : Nq != Nk)) return FA_ERR_UNSUPPORTED;
  // Tensor element counts must fit the kernels' index arithmetic.
  const double qe = (double)B * Hq * Nq * d, ke = (double)B * Hkv * Nk * d;
  if (qe > 4.0e12 || ke > 4.0e12) return FA_ERR_UNSUPPORTED;
  if ((double)B * Hq > 2147483647.0 || Nq > (1 << 28) || Nk > (1 << 28))
    return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// Dropout probability -> keep threshold floor(p * 2^32) and 1 / (1 - p);
// FA_ERR_INVALID_ARG unless 0 <= p < 1.
int dropout_params(float p_drop, unsigned long long seed, unsigned long long offset, AttnArgs &a) {
  if (!(p_drop >= 0.f) || !(p_drop < 1.f)) return FA_ERR_INVALID_ARG;
  const double t = floor((double)p_drop * 4294967296.0);
  a.drop_thr = t >= 4294967295.0 ? 0xFFFFFFFFu : (uint32_t)t;
  a.drop_scale = (float)(1.0 / (1.0 - (double)p_drop));
  a.seed = seed;
  a.drop_offset = offset;
  return FA_OK;
}

int prologue(int *dev, AttnArgs &a) {
  int st = current_device_checked(dev);
  if (st) return st;
  st = check_arch(*dev);
  if (st) return st;
  a.err = error_word(*dev);
  return a.err ? FA_OK : FA_ERR_CUDA;
}

// One CTA, one barrier nobody arrives at: the bounded wait must expire.
__global__ void wait_selftest_kernel(long long limit_ns, unsigned *err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  WaitCtx w{err, &abort_flag, limit_ns};
  if (threadIdx.x == 0) (void)bounded_wait(smem_u32(&bar), 0, w);
  __syncthreads();
}

}  // namespace

int validate_sizes(int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal) {
  return check_sizes(B, Hq, Hkv, Nq, Nk, d, scale, causal);
}

int device_prologue(int *dev, AttnArgs &a) { return prologue(dev, a); }

int launch_wait_selftest(long long timeout_ns, cudaStream_t stream, unsigned *err) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(timeout_ns, err);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

EncodeTiledFn get_encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

}  // namespace fa

using fa::AttnArgs;

#define FA_EXPORT __attribute__((visibility("default")))

extern "C" {

FA_EXPORT const char *fa_strerror(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument (null pointer, size <= 0, Hq % Hkv != 0 or bad scale)";
    case FA_ERR_UNSUPPORTED: return "unsupported configuration (head dim, causal query/key lengths, or size)";
    case FA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case FA_ERR_ARCH: return "device is not compute capability 10.0 (sm_100a build)";
    case FA_ERR_CUDA: return "CUDA runtime error or kernel launch failure";
    case FA_ERR_TIMEOUT: return "a bounded in-kernel wait expired";
    default: return "unknown status";
  }
}

FA_EXPORT size_t fa_bwd_workspace_size(int B, int Hq, int Nq, int d) {
  if (B <= 0 || Hq <= 0 || Nq <= 0 || d <= 0) return 0;
  return fa::ws_bytes(B, Hq, Nq, d);
}

FA_EXPORT int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
           int Hkv, int Nq, int Nk, int d, float scale, int causal, fa_stream_t stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  int st = fa::check_sizes(B, Hq, Hkv, Nq, Nk, d, scale, causal);
  if (st) return st;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (!fa::aligned16(q) || !fa::aligned16(k) || !fa::aligned16(v) || !fa::aligned16(o) ||
      !fa::aligned16(lse))
    return FA_ERR_ALIGNMENT;
  AttnArgs a;
  int dev;
  if ((st = fa::prologue(&dev, a))) return st;
  a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Nq = Nq; a.Nk = Nk; a.d = d;
  a.scale = scale; a.causal = causal ? 1 : 0; a.stream = (cudaStream_t)stream;
  return fa::launch_fwd_bf16_sm100(a);
}

FA_EXPORT int fa_fwd_pair(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                          int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                          fa_stream_t stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  int st = fa::check_sizes(B, Hq, Hkv, Nq, Nk, d, scale, causal);
  if (st) return st;
  if (d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (!fa::aligned16(q) || !fa::aligned16(k) || !fa::aligned16(v) || !fa::aligned16(o) ||
      !fa::aligned16(lse))
    return FA_ERR_ALIGNMENT;
  AttnArgs a;
  int dev;
  if ((st = fa::prologue(&dev, a))) return st;
  a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Nq = Nq; a.Nk = Nk; a.d = d;
  a.scale = scale; a.causal = causal ? 1 : 0; a.stream = (cudaStream_t)stream;
  return fa::launch_fwd_pair_bf16_sm100(a);
}

FA_EXPORT int fa_fwd_splitkv_num_splits(int B, int Hq, int Nq, int Nk, int d) {
  if (B <= 0 || Hq <= 0 || Nq <= 0 || Nk <= 0) return 0;
  if (d != 64 && d != 128 && d != 256) return 0;
  // Units of the plain forward (query blocks of 256 rows, 128 at d = 256);
  // split the key range so that one wave of 148 SMs is as full as it gets
  // without a second, partial wave (measured best on B200: B1 H8 Nq512
  // Nk16384 d128 runs 52 us with 9 pieces, 67 us with 19), keeping at least
  // two 128-key blocks per piece.
  const long long rows_per_unit = d == 256 ? 128 : 256;
  const long long units = (long long)B * Hq * ((Nq + rows_per_unit - 1) / rows_per_unit);
  const long long kblocks = (Nk + 127) / 128;
  long long s = 148 / units;
  s = s < kblocks / 2 ? s : kblocks / 2;
  s = s < 64 ? s : 64;
  return s < 1 ? 1 : (int)s;
}

FA_EXPORT size_t fa_fwd_splitkv_workspace_size(int B, int Hq, int Nq, int d, int num_splits) {
  if (B <= 0 || Hq <= 0 || Nq <= 0 || d <= 0 || num_splits <= 0) return 0;
  if (num_splits == 1) return 0;
  return fa::splitkv_ws_bytes(num_splits, B, Hq, Nq, d);
}

FA_EXPORT int fa_fwd_splitkv(const void *q, const void *k, const void *v, void *o, float *lse,
                             void *workspace, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                             float scale, int causal, int num_splits, fa_stream_t stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (num_splits <= 0 || num_splits > 1024) return FA_ERR_INVALID_ARG;
  if (num_splits > 1 && !workspace) return FA_ERR_INVALID_ARG;
  int st = fa::check_sizes(B, Hq, Hkv, Nq, Nk, d, scale, causal, true);
  if (st) return st;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (!fa::aligned16(q) || !fa::aligned16(k) || !fa::aligned16(v) || !fa::aligned16(o) ||
      !fa::aligned16(lse))
    return FA_ERR_ALIGNMENT;
  if (num_splits > 1 && ((uintptr_t)workspace & 255u)) return FA_ERR_ALIGNMENT;
  AttnArgs a;
  int dev;
  if ((st = fa::prologue(&dev, a))) return st;
  a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse; a.ws = workspace;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Nq = Nq; a.Nk = Nk; a.d = d;
  a.scale = scale; a.causal = causal ? 1 : 0; a.stream = (cudaStream_t)stream;
  a.causal_off = causal ? Nk - Nq : 0;
  a.splits = num_splits;
  return fa::launch_fwd_splitkv_bf16_sm100(a);
}

FA_EXPORT int fa_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
           const void *dout, void *dq, void *dk, void *dv, void *workspace, int B, int Hq,
           int Hkv, int Nq, int Nk, int d, float scale, int causal, fa_stream_t stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace)
    return FA_ERR_INVALID_ARG;
  int st = fa::check_sizes(B, Hq, Hkv, Nq, Nk, d, scale, causal);
  if (st) return st;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  const void *ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv};
  for (const void *p : ptrs)
    if (!fa::aligned16(p)) return FA_ERR_ALIGNMENT;
  if (((uintptr_t)workspace & 255u) != 0) return FA_ERR_ALIGNMENT;
  AttnArgs a;
  int dev;
  if ((st = fa::prologue(&dev, a))) return st;
  a.q = q; a.k = k; a.v = v; a.o_in = o; a.lse = const_cast<float *>(lse); a.dout = dout;
  a.dq = dq; a.dk = dk; a.dv = dv; a.ws = workspace;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Nq = Nq; a.Nk = Nk; a.d = d;
  a.scale = scale; a.causal = causal ? 1 : 0; a.stream = (cudaStream_t)stream;
  return fa::launch_bwd_bf16_sm100(a);
}

FA_EXPORT int fa_fwd_dropout(const void *q, const void *k, const void *v, void *o, float *lse,
                             int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                             float p_drop, unsigned long long seed, unsigned long long offset,
                             fa_stream_t stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  AttnArgs a;
  int st = fa::dropout_params(p_drop, seed, offset, a);
  if (st) return st;
  if ((st = fa::check_sizes(B, Hq, Hkv, Nq, Nk, d, scale, causal))) return st;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (!fa::aligned16(q) || !fa::aligned16(k) || !fa::aligned16(v) || !fa::aligned16(o) ||
      !fa::aligned16(lse))
    return FA_ERR_ALIGNMENT;
  int dev;
  if ((st = fa::prologue(&dev, a))) return st;
  a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Nq = Nq; a.Nk = Nk; a.d = d;
  a.scale = scale; a.causal = causal ? 1 : 0; a.stream = (cudaStream_t)stream;
  return fa::launch_fwd_bf16_sm100(a);
}

FA_EXPORT int fa_fwd_fp8(const void *q, const void *k, const void *v, void *o, float *lse,
                         int B, int Hq, int Hkv, int N, int d, float scale, float descale_q,
                         float descale_k, float descale_v, int causal, fa_stream_t stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  const float ds[3] = {descale_q, descale_k, descale_v};
  for (float x : ds)
    if (!(x > 0.f) || !isfinite(x)) return FA_ERR_INVALID_ARG;
  int st = fa::check_sizes(B, Hq, Hkv, N, N, d, scale, causal);
  if (st) return st;
  if (d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (!fa::aligned16(q) || !fa::aligned16(k) || !fa::aligned16(v) || !fa::aligned16(o) ||
      !fa::aligned16(lse))
    return FA_ERR_ALIGNMENT;
  AttnArgs a;
  int dev;
  if ((st = fa::prologue(&dev, a))) return st;
  a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Nq = N; a.Nk = N; a.d = d;
  a.scale = scale; a.causal = causal ? 1 : 0; a.stream = (cudaStream_t)stream;
  a.descale_q = descale_q; a.descale_k = descale_k; a.descale_v = descale_v;
  return fa::launch_fwd_e4m3_sm100(a);
}

FA_EXPORT int fa_bwd_dropout(const void *q, const void *k, const void *v, const void *o,
                             const float *lse, const void *dout, void *dq, void *dk, void *dv,
                             void *workspace, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                             float scale, int causal, float p_drop, unsigned long long seed,
                             unsigned long long offset, fa_stream_t stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace)
    return FA_ERR_INVALID_ARG;
  AttnArgs a;
  int st = fa::dropout_params(p_drop, seed, offset, a);
  if (st) return st;
  if ((st = fa::check_sizes(B, Hq, Hkv, Nq, Nk, d, scale, causal))) return st;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  const void *ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv};
  for (const void *p : ptrs)
    if (!fa::aligned16(p)) return FA_ERR_ALIGNMENT;
  if (((uintptr_t)workspace & 255u) != 0) return FA_ERR_ALIGNMENT;
  int dev;
  if ((st = fa::prologue(&dev, a))) return st;
  a.q = q; a.k = k; a.v = v; a.o_in = o; a.lse = const_cast<float *>(lse); a.dout = dout;
  a.dq = dq; a.dk = dk; a.dv = dv; a.ws = workspace;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Nq = Nq; a.Nk = Nk; a.d = d;
  a.scale = scale; a.causal = causal ? 1 : 0; a.stream = (cudaStream_t)stream;
  return fa::launch_bwd_bf16_sm100(a);
}

FA_EXPORT int fa_bwd_prep(const void *q, const void *k, const void *o, const float *lse,
                          const void *dout, void *workspace, int B, int Hq, int Hkv, int Nq,
                          int Nk, int d, float scale, fa_stream_t stream) {
  if (!q || !k || !o || !lse || !dout || !workspace) return FA_ERR_INVALID_ARG;
  int st = fa::check_sizes(B, Hq, Hkv, Nq, Nk, d, scale, 0);
  if (st) return st;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  const void *ptrs[] = {q, k, o, lse, dout};
  for (const void *p : ptrs)
    if (!fa::aligned16(p)) return FA_ERR_ALIGNMENT;
  if (((uintptr_t)workspace & 255u) != 0) return FA_ERR_ALIGNMENT;
  AttnArgs a;
  int dev;
  if ((st = fa::prologue(&dev, a))) return st;
  a.q = q; a.k = k; a.o_in = o; a.lse = const_cast<float *>(lse); a.dout = dout; a.ws = workspace;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Nq = Nq; a.Nk = Nk; a.d = d; a.scale = scale;
  a.stream = (cudaStream_t)stream;
  return fa::launch_bwd_prep_bf16(a);
}

FA_EXPORT int fa_bwd_dkdv(const void *q, const void *k, const void *v, const void *dout,
                          void *dk, void *dv, void *workspace, int B, int Hq, int Hkv, int Nq,
                          int Nk, int d, float scale, int causal, fa_stream_t stream) {
  if (!q || !k || !v || !dout || !dk || !dv || !workspace) return FA_ERR_INVALID_ARG;
  int st = fa::check_sizes(B, Hq, Hkv, Nq, Nk, d, scale, causal);
  if (st) return st;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  const void *ptrs[] = {q, k, v, dout, dk, dv};
  for (const void *p : ptrs)
    if (!fa::aligned16(p)) return FA_ERR_ALIGNMENT;
  if (((uintptr_t)workspace & 255u) != 0) return FA_ERR_ALIGNMENT;
  AttnArgs a;
  int dev;
  if ((st = fa::prologue(&dev, a))) return st;
  a.q = q; a.k = k; a.v = v; a.dout = dout; a.dk = dk; a.dv = dv; a.ws = workspace;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Nq = Nq; a.Nk = Nk; a.d = d;
  a.scale = scale; a.causal = causal ? 1 : 0; a.stream = (cudaStream_t)stream;
  return fa::launch_bwd_dkdv_bf16_sm100(a);
}

FA_EXPORT int fa_bwd_dq(const void *workspace, void *dq, int B, int Hq, int Nq, int d,
                        float scale, fa_stream_t stream) {
  if (!workspace || !dq) return FA_ERR_INVALID_ARG;
  int st = fa::check_sizes(B, Hq, Hq, Nq, Nq, d, scale, 0);
  if (st) return st;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (!fa::aligned16(dq) || ((uintptr_t)workspace & 255u) != 0) return FA_ERR_ALIGNMENT;
  AttnArgs a;
  int dev;
  if ((st = fa::prologue(&dev, a))) return st;
  a.ws = const_cast<void *>(workspace); a.dq = dq;
  a.B = B; a.Hq = Hq; a.Hkv = Hq; a.Nq = Nq; a.Nk = Nq; a.d = d; a.scale = scale;
  a.stream = (cudaStream_t)stream;
  return fa::launch_bwd_dq_bf16(a);
}

FA_EXPORT int fa_fwd_f32(const float *q, const float *k, const float *v, float *o, float *lse, int B,
               int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
               fa_stream_t stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  int st = fa::check_sizes(B, Hq, Hkv, Nq, Nk, d, scale, causal);
  if (st) return st;
  if (d > 256 || d % 4 != 0) return FA_ERR_UNSUPPORTED;
  if (!fa::aligned16(q) || !fa::aligned16(k) || !fa::aligned16(v) || !fa::aligned16(o) ||
      !fa::aligned16(lse))
    return FA_ERR_ALIGNMENT;
  AttnArgs a;
  int dev;
  if ((st = fa::prologue(&dev, a))) return st;
  a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Nq = Nq; a.Nk = Nk; a.d = d;
  a.scale = scale; a.causal = causal ? 1 : 0; a.stream = (cudaStream_t)stream;
  return fa::launch_fwd_f32(a);
}

FA_EXPORT int fa_bwd_f32(const float *q, const float *k, const float *v, const float *o, const float *lse,
               const float *dout, float *dq, float *dk, float *dv, void *workspace, int B,
               int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
               fa_stream_t stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace)
    return FA_ERR_INVALID_ARG;
  int st = fa::check_sizes(B, Hq, Hkv, Nq, Nk, d, scale, causal);
  if (st) return st;
  if (d > 256 || d % 4 != 0) return FA_ERR_UNSUPPORTED;
  const void *ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv};
  for (const void *p : ptrs)
    if (!fa::aligned16(p)) return FA_ERR_ALIGNMENT;
  if (((uintptr_t)workspace & 255u) != 0) return FA_ERR_ALIGNMENT;
  AttnArgs a;
  int dev;
  if ((st = fa::prologue(&dev, a))) return st;
  a.q = q; a.k = k; a.v = v; a.o_in = o; a.lse = const_cast<float *>(lse); a.dout = dout;
  a.dq = dq; a.dk = dk; a.dv = dv; a.ws = workspace;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Nq = Nq; a.Nk = Nk; a.d = d;
  a.scale = scale; a.causal = causal ? 1 : 0; a.stream = (cudaStream_t)stream;
  return fa::launch_bwd_f32(a);
}

FA_EXPORT int fa_device_status(fa_stream_t stream) {
  int dev;
  int st = fa::current_device_checked(&dev);
  if (st) return st;
  unsigned *err = fa::error_word(dev);
  if (!err) return FA_ERR_CUDA;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return FA_ERR_CUDA;
  unsigned host = 0, zero = 0;
  if (cudaMemcpy(&host, err, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess)
    return FA_ERR_CUDA;
  if (host && cudaMemcpy(err, &zero, sizeof(unsigned), cudaMemcpyHostToDevice) != cudaSuccess)
    return FA_ERR_CUDA;
  if (host & fa::kErrTimeout) return FA_ERR_TIMEOUT;
  return host ? FA_ERR_CUDA : FA_OK;
}

FA_EXPORT int fa_wait_selftest(long long timeout_ns, fa_stream_t stream) {
  if (timeout_ns < 1 || timeout_ns > 1000000000LL) return FA_ERR_INVALID_ARG;
  AttnArgs a;
  int dev;
  int st = fa::prologue(&dev, a);
  if (st) return st;
  return fa::launch_wait_selftest(timeout_ns, (cudaStream_t)stream, a.err);
}

}  // extern "C"
