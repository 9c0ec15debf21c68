// fa_noalloc.cu -- fa_bwd_noalloc: the BF16 backward without a caller
// workspace.
//
// fa_bwd needs scratch device memory (the row vector D and the f32 dQ
// accumulator) and asks the caller to allocate it.  Some callers cannot
// allocate device memory where they call the backward: a plugin inside a
// host application that owns the device memory pool and does not let
// plugins call cudaMalloc, or a latency-critical loop where cudaMalloc's
// possible implicit device synchronisation is not acceptable.  For them this
// file keeps the scratch in one fixed array in the library's device image,
// sized kNoAllocScratchBytes.
//
// The first fa_bwd_noalloc call on a device looks up the array's device
// address (cudaGetSymbolAddress, with that device current) and caches it.
// The runtime loads device code lazily, so that lookup is also what creates
// the array on the device: the first call makes a 32 MiB allocation inside
// the runtime, may synchronise the device and fails with FA_ERR_CUDA when the
// memory is not there.  Make that first call during set-up, before any stream
// capture; the array then stays on the device until the process exits.  The
// cached address is that of the device's primary context and goes stale after
// cudaDeviceReset (as does the error-word address of fa_capi.cu).  All calls
// share the one array and leave their contents in it: the kernels zero the
// dQ accumulator and rewrite D on every call, and two calls whose kernels
// overlap on the GPU (different streams, or different host threads on one
// device) race on it.
#include <atomic>

#include "../../include/fa.h"
#include "common.cuh"
#include "launch.h"

// 32 MiB: the backward scratch is about 4*B*Hq*(Nq*(d + 2) + d) bytes (plus
// padding), so this covers e.g. B*Hq*Nq <= 64,000 query rows at d = 128.
static constexpr size_t kNoAllocScratchBytes = (size_t)32 << 20;
static __device__ __align__(256) unsigned char fa_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::atomic<void *> g_scratch_addr[kMaxDevices];

// Device address of fa_noalloc_scratch on device `dev` (current), looked up
// once per device.  The host-side symbol itself is not a device address.
void *scratch_on_device(int dev) {
  void *p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p) return p;
  if (cudaGetSymbolAddress(&p, fa_noalloc_scratch) != cudaSuccess || !p) return nullptr;
  g_scratch_addr[dev].store(p, std::memory_order_release);
  return p;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" __attribute__((visibility("default"))) int fa_bwd_noalloc(
    const void *q, const void *k, const void *v, const void *o, const float *lse,
    const void *dout, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int Nq, int Nk,
    int d, float scale, int causal, fa_stream_t stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  int st = fa::validate_sizes(B, Hq, Hkv, Nq, Nk, d, scale, causal);
  if (st) return st;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  const void *ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv};
  for (const void *p : ptrs)
    if (!aligned16(p)) return FA_ERR_ALIGNMENT;
  // Scratch needed for this problem; refuse (before touching the device)
  // anything the fixed array cannot hold.
  const double need = (double)fa::ws_bytes(B, Hq, Nq, d);
  if (need > (double)kNoAllocScratchBytes) return FA_ERR_UNSUPPORTED;
  fa::AttnArgs a;
  int dev;
  if ((st = fa::device_prologue(&dev, a))) return st;
  void *scratch = scratch_on_device(dev);
  if (!scratch) return FA_ERR_CUDA;
  a.q = q; a.k = k; a.v = v; a.o_in = o; a.lse = const_cast<float *>(lse); a.dout = dout;
  a.dq = dq; a.dk = dk; a.dv = dv; a.ws = scratch;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Nq = Nq; a.Nk = Nk; a.d = d;
  a.scale = scale; a.causal = causal ? 1 : 0; a.stream = (cudaStream_t)stream;
  return fa::launch_bwd_bf16_sm100(a);
}
