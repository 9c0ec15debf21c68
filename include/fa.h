/*
 * fa.h -- C ABI of the exact-attention library (libfa.so), sm_100a only.
 *
 * The operation (FlashAttention blog, ruizhehou.github.io, section 1 and
 * section 3; CSDN FlashAttention-1 tutorial, section 1):
 *
 *     S = scale * Q K^T      (causal: S_ij = -inf for j > i, top-left aligned,
 *                             the is_causal=True option of the blog's
 *                             section 5 call)
 *     P = softmax(S)         row-wise, max-subtracted (blog section 2.2)
 *     O = P V
 *     L_i = m_i + ln(l_i)    per-row log-sum-exp of the scaled scores, natural
 *                            log (the blog's section 2.3 saves m and l per row;
 *                            this library saves the one number L)
 *
 * Forward: the tiled online-softmax recurrence with deferred normalisation
 * (blog section 4.1, "v2"; CSDN tutorial section 3).  Backward: P is
 * recomputed from Q, K and L rather than stored (blog section 2.3); the
 * gradients are those of f = sum(O * dO).
 *
 * Layout (every tensor dense, row-major, d fastest):
 *     q, o, dout, dq : [B, Hq,  Nq, d]
 *     k, v, dk, dv   : [B, Hkv, Nk, d]
 *     lse            : [B, Hq,  Nq] float32
 * Grouped-query attention (wiki "FlashAttention", FlashAttention-2 history):
 * query head h reads key/value head h / (Hq / Hkv); dk and dv of a key/value
 * head are the sums over its query heads.
 *
 * Ownership: the caller allocates every buffer (inputs, outputs, workspace)
 * in device memory.  Inputs are read only; outputs are fully overwritten.
 * The library allocates nothing, keeps no per-call state and never
 * synchronises the host with the device: work is enqueued on `stream` and
 * the call returns.  Asynchronous execution errors surface at the caller's
 * next synchronisation, as for any CUDA call.
 *
 * Errors: every entry point returns an fa_status; nothing is printed, thrown
 * or aborted.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st *fa_stream_t;

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null pointer, size <= 0, Hq % Hkv != 0, scale not finite or <= 0 */
  FA_ERR_UNSUPPORTED = 2, /* head dim, length or mask combination the library does not run */
  FA_ERR_ALIGNMENT = 3,   /* a pointer is not 16-byte aligned */
  FA_ERR_ARCH = 4,        /* current device is not compute capability 10.0 */
  FA_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed */
  FA_ERR_TIMEOUT = 6      /* a bounded in-kernel wait expired (reported by fa_device_status) */
} fa_status;

/*
 * fa_fwd -- BF16 forward: O and L of the operation above, computed tile by
 * tile with the online softmax and one final normalisation (blog section 4.1
 * "v2", CSDN tutorial section 3).  q, k, v, o: bfloat16; lse: float32.
 * d must be 64, 128 or 256.  causal != 0 requires Nq == Nk.
 * Nq, Nk >= 1 (any length; tails are masked).  scale is applied to Q K^T
 * before the softmax (1/sqrt(d) for standard attention).
 * Returns FA_ERR_UNSUPPORTED for other head dims, FA_ERR_ALIGNMENT when a
 * pointer is not 16-byte aligned.
 */
int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
           int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
           fa_stream_t stream);

/*
 * fa_fwd_pair -- fa_fwd computed by pairs of CTAs on neighbouring SMs that
 * share each tile's tensor-core MMAs (tcgen05 cta_group::2, M = 256: the
 * two-CTA MMA the wiki's FlashAttention-4 paragraph lists).  Each CTA of a
 * pair holds its own 128-row Q tiles and loads half of every K tile (64 of
 * the 128 keys) and half of every V tile (d / 2 of the columns), so a pair
 * moves each K/V block into shared memory once instead of twice.  Same
 * arguments, layouts, result and errors as fa_fwd; d must be 128 or 256
 * (FA_ERR_UNSUPPORTED otherwise).  fa_fwd keeps the single-CTA kernels,
 * which measured 20-35% faster on B200 at d = 128 and 256, causal or not.
 */
int fa_fwd_pair(const void *q, const void *k, const void *v, void *o, float *lse,
                int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                fa_stream_t stream);

/*
 * Split-KV forward for inference shapes -- few query rows per head against a
 * long key range (the FlashAttention blog, section 4.2, on batch-1 inference
 * leaving the GPU idle when only batch and heads are parallel).  The visible
 * key range of each 256-row query block (128 at d = 256) is cut into
 * num_splits contiguous pieces of 128-key blocks, one CTA per piece; each
 * piece's normalised output O_s (float32) and log-sum-exp L_s go to the
 * workspace and a second kernel merges them:
 *     L = log sum_s exp(L_s),   O = sum_s exp(L_s - L) O_s   -> bf16,
 * the identity the online softmax uses to combine two blocks (blog section
 * 2.2).  A piece that sees no key of a row has L_s = -inf and adds nothing.
 *
 * Causal here is bottom-right aligned: the Nq queries are the last Nq
 * positions of the sequence, key j is hidden from query i when
 * j > i + (Nk - Nq); Nq <= Nk is required (FA_ERR_UNSUPPORTED otherwise).
 * For Nq == Nk this is fa_fwd's mask.
 *
 * fa_fwd_splitkv_num_splits -- a piece count that fills one wave of the
 *   GPU's 148 SMs (1 when the query blocks alone do; 0 for invalid sizes).
 * fa_fwd_splitkv_workspace_size -- bytes of workspace for num_splits pieces:
 *   float32 [num_splits][B][Hq][Nq][d] then, 256-byte aligned,
 *   [num_splits][B][Hq][Nq]; 0 when num_splits == 1 (no workspace needed) or
 *   a size is invalid.
 * fa_fwd_splitkv -- tensors, dtypes and layouts as fa_fwd; workspace: at
 *   least fa_fwd_splitkv_workspace_size(...) bytes, 256-byte aligned, may be
 *   NULL when num_splits == 1; 1 <= num_splits <= 1024 (more pieces than key
 *   blocks leave some empty), else FA_ERR_INVALID_ARG.
 */
int fa_fwd_splitkv_num_splits(int B, int Hq, int Nq, int Nk, int d);
size_t fa_fwd_splitkv_workspace_size(int B, int Hq, int Nq, int d, int num_splits);
int fa_fwd_splitkv(const void *q, const void *k, const void *v, void *o, float *lse,
                   void *workspace, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                   int causal, int num_splits, fa_stream_t stream);

/*
 * Dropout on P (BF16).  The blog's section 5 call passes dropout_p to
 * F.scaled_dot_product_attention (0 there); these entry points take p > 0:
 *     O = (P * Z) V / (1 - p),   L = log-sum-exp of the undropped scores,
 * with Z_ij = 1 when word (j mod 4) of Philox4x32-10 (Salmon et al.,
 * "Parallel random numbers: as easy as 1, 2, 3", SC 2011) with
 *     key     = (seed mod 2^32, seed >> 32),
 *     counter = (j / 4, i, b*Hq + h, offset mod 2^32)
 * is >= floor(p * 2^32), else 0 (i query row, j key column, h query head).
 * The mask is a pure function of (seed, offset, b, h, i, j): fa_bwd_dropout
 * with the same seed and offset regenerates it.  Gradients of
 * f = sum(O * dO): dV = (P*Z)^T dO / (1-p), dP = (dO V^T) * Z / (1-p),
 * dS = P * (dP - D) with D = rowsum(dO * O).
 *
 * Same tensors, layouts, size rules and errors as fa_fwd / fa_bwd, plus:
 * 0 <= p_drop < 1 (else FA_ERR_INVALID_ARG); p_drop = 0 computes exactly
 * fa_fwd / fa_bwd.  Both support d = 64, 128 and 256.
 */
int fa_fwd_dropout(const void *q, const void *k, const void *v, void *o, float *lse,
                   int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                   float p_drop, unsigned long long seed, unsigned long long offset,
                   fa_stream_t stream);
int fa_bwd_dropout(const void *q, const void *k, const void *v, const void *o, const float *lse,
                   const void *dout, void *dq, void *dk, void *dv, void *workspace,
                   int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                   float p_drop, unsigned long long seed, unsigned long long offset,
                   fa_stream_t stream);

/*
 * fa_fwd_fp8 -- attention forward on FP8 inputs.  The wiki's FlashAttention-3
 * paragraph ("FlashAttention", newton.com.tw) names low-precision FP8 as one
 * of the Hopper features FA3 uses and defines nothing further; this entry
 * point reads it as: Q, K, V hold OCP FP8 E4M3 codes (one byte per element:
 * sign, 4 exponent bits with bias 7, 3 mantissa bits; largest finite 448),
 * each tensor with one dequantisation factor, so the tensors meant are
 * descale_q * Q^, descale_k * K^, descale_v * V^ (code values Q^ ...), and
 *     O = softmax(scale * (descale_q Q^)(descale_k K^)^T [+ causal]) (descale_v V^),
 *     L = log-sum-exp of the scaled scores (natural log, float32),
 * the same quantity as fa_fwd computes for those tensors.  S accumulates in
 * float32 on the tensor cores; P is rounded to e4m3 for the P V product,
 * stored as 2^4 * exp(s - m) with m a running row maximum that lags by less
 * than a factor 2^4, so stored values are at most 256: the rounding error is
 * at most 2^-4 of the value from 2^-6 up and at most 2^-10 below (the
 * subnormal range).  O is accumulated in float32 and written as bf16.
 *
 * q [B, Hq, N, d], k and v [B, Hkv, N, d]: E4M3 codes, contiguous, 16-byte
 * aligned; o [B, Hq, N, d] bf16 and lse [B, Hq, N] float32 written by the
 * call (caller-owned device memory).  Nq = Nk = N; causal is top-left.
 * descale_*: finite and > 0 (else FA_ERR_INVALID_ARG).  d = 128 or 256
 * (FA_ERR_UNSUPPORTED otherwise).  Other size rules and errors as fa_fwd.
 * Code values that are NaN (S.1111.111) give NaN outputs for the rows they
 * reach.
 */
int fa_fwd_fp8(const void *q, const void *k, const void *v, void *o, float *lse,
               int B, int Hq, int Hkv, int N, int d, float scale,
               float descale_q, float descale_k, float descale_v, int causal,
               fa_stream_t stream);

/*
 * fa_bwd_workspace_size -- bytes of device workspace fa_bwd and fa_bwd_f32
 * need, i.e. what the recomputing backward (blog section 2.3) keeps besides
 * the inputs (float32 throughout): the per-row vector D = rowsum(dO * O) and the
 * per-row base-2 log-sum-exp used by the backward, each padded to a multiple
 * of 128 rows per head; one centring vector per head (B*Hq*d); a work
 * counter of the persistent main pass; and a dQ accumulator (B*Hq*Nq*d),
 * 256-byte aligned.  About 4*B*Hq*(Nq*(d+2) + d) + 256 bytes.  Returns 0 for
 * invalid sizes.
 */
size_t fa_bwd_workspace_size(int B, int Hq, int Nq, int d);

/*
 * fa_bwd -- BF16 backward: dQ, dK, dV of f = sum(O * dO) with P recomputed
 * from Q, K and L instead of stored (blog section 2.3): dV = P^T dO,
 * dP = dO V^T, dS = P * (dP - D) with D = rowsum(dO * O), dQ = scale dS K,
 * dK = scale dS^T Q.  q, k, v, o, dout: bfloat16 (o and lse as written
 * by fa_fwd for the same inputs); dq, dk, dv: bfloat16 outputs; workspace:
 * at least fa_bwd_workspace_size(B, Hq, Nq, d) bytes of device memory,
 * 256-byte aligned, contents ignored on entry and clobbered.
 * Same size rules as fa_fwd.
 */
int fa_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
           const void *dout, void *dq, void *dk, void *dv, void *workspace,
           int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
           fa_stream_t stream);

/*
 * The three stages fa_bwd runs, exposed so a caller can time or schedule
 * them separately.  Called in this order on one stream with the same
 * workspace they compute exactly what fa_bwd computes (BF16 only):
 *   fa_bwd_prep  -- per key/value head the centring vector c (the mean of its
 *                   first 64 key rows, rounded to integers); per query row
 *                   D = rowsum(dout * o) and the base-2 log-sum-exp shifted
 *                   by scale * q . c; the dQ accumulator and the main pass's
 *                   work counter zeroed;
 *   fa_bwd_dkdv  -- the main pass: dk, dv written, dQ accumulated (f32) in
 *                   the workspace.  Needs fa_bwd_prep on the same workspace
 *                   before every call (d = 64 and 128 hand out work units
 *                   through the counter prep zeroes);
 *   fa_bwd_dq    -- dq = bf16(scale * accumulator).
 * Same argument rules as fa_bwd.
 */
int fa_bwd_prep(const void *q, const void *k, const void *o, const float *lse, const void *dout,
                void *workspace, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                fa_stream_t stream);
int fa_bwd_dkdv(const void *q, const void *k, const void *v, const void *dout, void *dk,
                void *dv, void *workspace, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                float scale, int causal, fa_stream_t stream);
int fa_bwd_dq(const void *workspace, void *dq, int B, int Hq, int Nq, int d, float scale,
              fa_stream_t stream);

/*
 * fa_fwd_f32 / fa_bwd_f32 -- the same operations with float32 q, k, v, o,
 * dout, dq, dk, dv (FP32 CUDA-core arithmetic; correctness path for float32
 * inputs).  d must be a multiple of 4 and <= 256.
 */
int fa_fwd_f32(const float *q, const float *k, const float *v, float *o, float *lse,
               int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
               fa_stream_t stream);
int fa_bwd_f32(const float *q, const float *k, const float *v, const float *o,
               const float *lse, const float *dout, float *dq, float *dk, float *dv,
               void *workspace, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
               int causal, fa_stream_t stream);

/*
 * fa_bwd_noalloc -- fa_bwd for callers that cannot allocate device memory
 * where they run the backward (for example a plugin inside an application
 * that owns the device memory pool, or a loop that must not risk the device
 * synchronisation cudaMalloc can cause).  Same arguments and results as
 * fa_bwd, minus the workspace: the scratch lives in one fixed 32 MiB array
 * inside the library, held on each GPU from the first call there until the
 * process exits.  The FlashAttention pages describe no such call; it is an
 * interface convenience.
 * Returns FA_ERR_UNSUPPORTED, without touching the device, when the problem
 * needs more scratch than that (about 4*B*Hq*(Nq*(d+2) + d) bytes plus
 * padding, e.g. more than about 64,000 query rows B*Hq*Nq at d = 128).
 * First call on a device: the CUDA runtime loads the library's device code
 * lazily, so the array is created then (a 32 MiB device allocation made by
 * the runtime, which can synchronise the device and can fail with FA_ERR_CUDA
 * when the device is out of memory) and its address is looked up and cached.
 * Make that first call during set-up, before any stream capture; later calls
 * allocate nothing and do not synchronise.  The cached address belongs to the
 * device's primary context: after cudaDeviceReset the library must be
 * reloaded (the same holds for the device error word of every entry point).
 * Every call uses the same array: calls whose kernels overlap on the GPU
 * (other streams or threads on the same device) race and must be ordered by
 * the caller.
 */
int fa_bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                   const float *lse, const void *dout, void *dq, void *dk, void *dv,
                   int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                   fa_stream_t stream);

/*
 * fa_device_status -- synchronises `stream`, then reads and clears the
 * library's device error word on the current device.  Returns FA_OK, or
 * FA_ERR_TIMEOUT when a kernel's bounded wait expired since the last call
 * (that kernel then returned early and its outputs are undefined), or
 * FA_ERR_CUDA when the synchronisation itself failed or a kernel refused to
 * run (its shared memory was not 1024-byte aligned).
 */
int fa_device_status(fa_stream_t stream);

/*
 * fa_wait_selftest -- launches one CTA that waits on a shared-memory barrier
 * nothing ever arrives at, with the library's bounded wait and a limit of
 * timeout_ns nanoseconds (1 .. 1e9).  The wait gives up, records
 * FA_ERR_TIMEOUT in the device error word and the kernel returns normally.
 * Exists so tests can show the timeout path ends cleanly; follow it with
 * fa_device_status.
 */
int fa_wait_selftest(long long timeout_ns, fa_stream_t stream);

/* fa_strerror -- static description of a status code. */
const char *fa_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
