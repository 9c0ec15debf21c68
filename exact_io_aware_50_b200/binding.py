"""ctypes binding of libfa.so -- argument marshalling only.

The ``fa_*`` functions mirror the C ABI one to one (raw device pointers as
ints, sizes, a CUDA stream handle) and return the status code.  ``forward``
and ``backward`` take torch CUDA tensors, allocate outputs/workspace with
torch (device memory only), pass pointers and torch's current stream, and
raise ``FaError`` on a non-zero status.  Every step of the computation runs in
the library's CUDA kernels; there is no other code path.
"""
from __future__ import annotations

import ctypes
import os

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_ALIGNMENT = 3
FA_ERR_ARCH = 4
FA_ERR_CUDA = 5
FA_ERR_TIMEOUT = 6

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libfa.so")
_lib = None

EXPORTS = ("fa_fwd", "fa_fwd_pair", "fa_fwd_fp8", "fa_fwd_dropout", "fa_bwd_dropout", "fa_fwd_splitkv",
           "fa_fwd_splitkv_num_splits",
           "fa_fwd_splitkv_workspace_size", "fa_bwd", "fa_bwd_workspace_size", "fa_bwd_prep",
           "fa_bwd_dkdv",
           "fa_bwd_dq", "fa_fwd_f32", "fa_bwd_f32", "fa_device_status", "fa_wait_selftest",
           "fa_strerror")


class FaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: status {status} ({fa_strerror(status)})")


def lib():
    """Load libfa.so (once).  Raises if the built library is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise RuntimeError(f"{lib_path} is missing: build it with "
                               "`python -m exact_io_aware_50_b200.build`")
        L = ctypes.CDLL(lib_path)
        P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        dims = [I, I, I, I, I, I, F, I, P]
        L.fa_fwd.argtypes = [P] * 5 + dims
        L.fa_fwd.restype = I
        L.fa_fwd_pair.argtypes = [P] * 5 + dims
        L.fa_fwd_pair.restype = I
        L.fa_fwd_f32.argtypes = [P] * 5 + dims
        L.fa_fwd_f32.restype = I
        U64 = ctypes.c_ulonglong
        L.fa_fwd_fp8.argtypes = [P] * 5 + [I, I, I, I, I, F, F, F, F, I, P]
        L.fa_fwd_fp8.restype = I
        L.fa_fwd_dropout.argtypes = [P] * 5 + [I, I, I, I, I, I, F, I, F, U64, U64, P]
        L.fa_fwd_dropout.restype = I
        L.fa_bwd_dropout.argtypes = [P] * 10 + [I, I, I, I, I, I, F, I, F, U64, U64, P]
        L.fa_bwd_dropout.restype = I
        L.fa_fwd_splitkv.argtypes = [P] * 6 + [I, I, I, I, I, I, F, I, I, P]
        L.fa_fwd_splitkv.restype = I
        L.fa_fwd_splitkv_num_splits.argtypes = [I] * 5
        L.fa_fwd_splitkv_num_splits.restype = I
        L.fa_fwd_splitkv_workspace_size.argtypes = [I] * 5
        L.fa_fwd_splitkv_workspace_size.restype = S
        L.fa_bwd.argtypes = [P] * 10 + dims
        L.fa_bwd.restype = I
        L.fa_bwd_f32.argtypes = [P] * 10 + dims
        L.fa_bwd_f32.restype = I
        L.fa_bwd_prep.argtypes = [P] * 6 + [I, I, I, I, I, I, F, P]
        L.fa_bwd_prep.restype = I
        L.fa_bwd_dkdv.argtypes = [P] * 7 + dims
        L.fa_bwd_dkdv.restype = I
        L.fa_bwd_dq.argtypes = [P, P, I, I, I, I, F, P]
        L.fa_bwd_dq.restype = I
        L.fa_bwd_workspace_size.argtypes = [I, I, I, I]
        L.fa_bwd_workspace_size.restype = S
        L.fa_device_status.argtypes = [P]
        L.fa_device_status.restype = I
        L.fa_wait_selftest.argtypes = [ctypes.c_longlong, P]
        L.fa_wait_selftest.restype = I
        L.fa_strerror.argtypes = [I]
        L.fa_strerror.restype = ctypes.c_char_p
        _lib = L
    return _lib


# ----------------------------------------------------------------- raw ABI
def fa_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, stream=0):
    return lib().fa_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, int(causal), stream)


def fa_fwd_pair(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, stream=0):
    return lib().fa_fwd_pair(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, int(causal), stream)


def fa_fwd_fp8(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, descale_q, descale_k, descale_v, causal,
               stream=0):
    return lib().fa_fwd_fp8(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, float(descale_q),
                            float(descale_k), float(descale_v), int(causal), stream)


def fa_fwd_dropout(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, p_drop, seed, offset,
                   stream=0):
    return lib().fa_fwd_dropout(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, int(causal),
                                float(p_drop), int(seed), int(offset), stream)


def fa_bwd_dropout(q, k, v, o, lse, dout, dq, dk, dv, ws, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                   p_drop, seed, offset, stream=0):
    return lib().fa_bwd_dropout(q, k, v, o, lse, dout, dq, dk, dv, ws, B, Hq, Hkv, Nq, Nk, d,
                                scale, int(causal), float(p_drop), int(seed), int(offset), stream)


def fa_fwd_splitkv(q, k, v, o, lse, ws, B, Hq, Hkv, Nq, Nk, d, scale, causal, num_splits,
                   stream=0):
    return lib().fa_fwd_splitkv(q, k, v, o, lse, ws, B, Hq, Hkv, Nq, Nk, d, scale, int(causal),
                                int(num_splits), stream)


def fa_fwd_splitkv_num_splits(B, Hq, Nq, Nk, d):
    return int(lib().fa_fwd_splitkv_num_splits(B, Hq, Nq, Nk, d))


def fa_fwd_splitkv_workspace_size(B, Hq, Nq, d, num_splits):
    return int(lib().fa_fwd_splitkv_workspace_size(B, Hq, Nq, d, num_splits))


def fa_fwd_f32(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, stream=0):
    return lib().fa_fwd_f32(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, int(causal), stream)


def fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, ws, B, Hq, Hkv, Nq, Nk, d, scale, causal, stream=0):
    return lib().fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, ws, B, Hq, Hkv, Nq, Nk, d, scale,
                        int(causal), stream)


def fa_bwd_f32(q, k, v, o, lse, dout, dq, dk, dv, ws, B, Hq, Hkv, Nq, Nk, d, scale, causal,
               stream=0):
    return lib().fa_bwd_f32(q, k, v, o, lse, dout, dq, dk, dv, ws, B, Hq, Hkv, Nq, Nk, d, scale,
                            int(causal), stream)


def fa_bwd_prep(q, k, o, lse, dout, ws, B, Hq, Hkv, Nq, Nk, d, scale, stream=0):
    return lib().fa_bwd_prep(q, k, o, lse, dout, ws, B, Hq, Hkv, Nq, Nk, d, scale, stream)


def fa_bwd_dkdv(q, k, v, dout, dk, dv, ws, B, Hq, Hkv, Nq, Nk, d, scale, causal, stream=0):
    return lib().fa_bwd_dkdv(q, k, v, dout, dk, dv, ws, B, Hq, Hkv, Nq, Nk, d, scale,
                             int(causal), stream)


def fa_bwd_dq(ws, dq, B, Hq, Nq, d, scale, stream=0):
    return lib().fa_bwd_dq(ws, dq, B, Hq, Nq, d, scale, stream)


def fa_bwd_workspace_size(B, Hq, Nq, d):
    return int(lib().fa_bwd_workspace_size(B, Hq, Nq, d))


def fa_device_status(stream=0):
    return lib().fa_device_status(stream)


def fa_wait_selftest(timeout_ns, stream=0):
    return lib().fa_wait_selftest(int(timeout_ns), stream)


def fa_strerror(status):
    try:
        return lib().fa_strerror(int(status)).decode()
    except RuntimeError:
        return "library not loaded"


# ----------------------------------------------------------- torch helpers
def _check(status, where):
    if status != FA_OK:
        raise FaError(status, where)


# Argument checks of the wrappers: shapes and dtypes first, then device and
# layout; each raises ValueError before the library is called.
def _check_qkv(where, q, k, v, dtypes):
    """q [B, Hq, Nq, d]; k, v [B, Hkv, Nk, d]; one dtype among `dtypes`."""
    if q.dim() != 4 or k.dim() != 4 or tuple(v.shape) != tuple(k.shape):
        raise ValueError(f"{where}: q must be [B, Hq, Nq, d] and k, v both [B, Hkv, Nk, d]")
    if q.shape[0] != k.shape[0] or q.shape[3] != k.shape[3]:
        raise ValueError(f"{where}: q and k disagree on B or d")
    if not (q.dtype == k.dtype == v.dtype) or q.dtype not in dtypes:
        raise ValueError(f"{where}: q, k, v must share one dtype among {tuple(map(str, dtypes))}")


def _check_bwd_in(where, q, o, lse, dout):
    """o and dout shaped and typed like q; lse float32 [B, Hq, Nq]."""
    import torch
    if tuple(o.shape) != tuple(q.shape) or tuple(dout.shape) != tuple(q.shape):
        raise ValueError(f"{where}: o and dout must have q's shape")
    if o.dtype != q.dtype or dout.dtype != q.dtype:
        raise ValueError(f"{where}: o and dout must have q's dtype")
    if tuple(lse.shape) != tuple(q.shape[:3]) or lse.dtype != torch.float32:
        raise ValueError(f"{where}: lse must be float32 [B, Hq, Nq]")


def _check_cuda(where, q, *others):
    """q and every other tensor: contiguous, on CUDA, and on q's device.  The
    library launches on the current device, which the wrappers set to q's
    (``_on``), so a tensor on another GPU would be read by kernels running on
    the wrong one."""
    for t in (q,) + others:
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{where}: inputs must be contiguous CUDA tensors")
        if t.device != q.device:
            raise ValueError(f"{where}: every tensor must be on q's device ({q.device}); "
                             f"got one on {t.device}")


def _on(q):
    """Context that makes q's device current for one library call."""
    import torch
    return torch.cuda.device(q.device)


def _workspace(where, workspace, B, Hq, Nq, d, device):
    """The caller's backward workspace, checked against fa_bwd_workspace_size
    (the C entry points take a bare pointer and cannot), or a new one."""
    import torch
    need = fa_bwd_workspace_size(B, Hq, Nq, d)
    if workspace is None:
        return torch.empty(need, device=device, dtype=torch.uint8)
    if (not workspace.is_cuda or not workspace.is_contiguous()
            or workspace.numel() * workspace.element_size() < need):
        raise ValueError(f"{where}: workspace must be a contiguous CUDA buffer of at least "
                         f"{need} bytes")
    if workspace.device != device:
        raise ValueError(f"{where}: workspace must be on q's device ({device}); "
                         f"got {workspace.device}")
    return workspace


def _shape(q, k):
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if Bk != B or dk != d:
        raise ValueError("q and k shapes disagree")
    return B, Hq, Hkv, Nq, Nk, d


def _stream(t):
    import torch
    return torch.cuda.current_stream(t.device).cuda_stream


def forward(q, k, v, scale=None, causal=False, out=None, lse=None, cta_pair=False):
    """O, L = attention(q, k, v) for contiguous CUDA tensors [B, H, N, d]
    (bf16 -> fa_fwd, or fa_fwd_pair with cta_pair=True; float32 ->
    fa_fwd_f32)."""
    import torch
    _check_qkv("forward", q, k, v, (torch.bfloat16, torch.float32))
    _check_cuda("forward", q, k, v)
    B, Hq, Hkv, Nq, Nk, d = _shape(q, k)
    scale = d ** -0.5 if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    L = torch.empty(B, Hq, Nq, device=q.device, dtype=torch.float32) if lse is None else lse
    if (tuple(o.shape) != tuple(q.shape) or o.dtype != q.dtype or tuple(L.shape) != (B, Hq, Nq)
            or L.dtype != torch.float32):
        raise ValueError("forward: out must be shaped and typed like q, lse float32 [B, Hq, Nq]")
    _check_cuda("forward", q, o, L)
    if cta_pair and q.dtype != torch.bfloat16:
        raise ValueError("forward: cta_pair=True needs bf16 tensors")
    fn = (fa_fwd_pair if cta_pair else fa_fwd) if q.dtype == torch.bfloat16 else fa_fwd_f32
    with _on(q):
        _check(fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), L.data_ptr(), B, Hq, Hkv,
                  Nq, Nk, d, scale, causal, _stream(q)), fn.__name__)
    return o, L


def forward_splitkv(q, k, v, scale=None, causal=False, num_splits=None, workspace=None):
    """O, L for bf16 q [B, Hq, Nq, d] against k, v [B, Hkv, Nk, d] with the key
    range cut into pieces merged by their log-sum-exp (fa_fwd_splitkv).
    Causal is bottom-right aligned (Nq <= Nk).  num_splits=None picks
    fa_fwd_splitkv_num_splits."""
    import torch
    _check_qkv("forward_splitkv", q, k, v, (torch.bfloat16,))
    _check_cuda("forward_splitkv", q, k, v)
    B, Hq, Hkv, Nq, Nk, d = _shape(q, k)
    scale = d ** -0.5 if scale is None else float(scale)
    if num_splits is None:
        num_splits = fa_fwd_splitkv_num_splits(B, Hq, Nq, Nk, d)
    need = max(fa_fwd_splitkv_workspace_size(B, Hq, Nq, d, num_splits), 1)
    if workspace is None:
        workspace = torch.empty(need, device=q.device, dtype=torch.uint8)
    elif (not workspace.is_cuda or not workspace.is_contiguous()
          or workspace.numel() * workspace.element_size() < need):
        raise ValueError(f"forward_splitkv: workspace must be a contiguous CUDA buffer of at "
                         f"least {need} bytes")
    elif workspace.device != q.device:
        raise ValueError(f"forward_splitkv: workspace must be on q's device ({q.device}); "
                         f"got {workspace.device}")
    o = torch.empty_like(q)
    L = torch.empty(B, Hq, Nq, device=q.device, dtype=torch.float32)
    with _on(q):
        _check(fa_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              L.data_ptr(), workspace.data_ptr(), B, Hq, Hkv, Nq, Nk, d, scale,
                              causal, num_splits, _stream(q)), "fa_fwd_splitkv")
    return o, L


def forward_fp8(q, k, v, descale_q, descale_k, descale_v, scale=None, causal=False):
    """O (bf16), L from E4M3 inputs (fa_fwd_fp8).  q, k, v: contiguous CUDA
    tensors of dtype float8_e4m3fn or uint8 (the codes); descale_*: the
    per-tensor dequantisation factors."""
    import torch
    _check_qkv("forward_fp8", q, k, v, (torch.float8_e4m3fn, torch.uint8))
    B, Hq, Hkv, Nq, Nk, d = _shape(q, k)
    if Nq != Nk:
        raise ValueError("forward_fp8: Nq must equal Nk")
    _check_cuda("forward_fp8", q, k, v)
    scale = d ** -0.5 if scale is None else float(scale)
    o = torch.empty(q.shape, device=q.device, dtype=torch.bfloat16)
    L = torch.empty(B, Hq, Nq, device=q.device, dtype=torch.float32)
    with _on(q):
        _check(fa_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), L.data_ptr(),
                          B, Hq, Hkv, Nq, d, scale, descale_q, descale_k, descale_v, causal,
                          _stream(q)), "fa_fwd_fp8")
    return o, L


def forward_dropout(q, k, v, p_drop, seed, offset=0, scale=None, causal=False):
    """O, L with dropout on P (bf16, fa_fwd_dropout)."""
    import torch
    _check_qkv("forward_dropout", q, k, v, (torch.bfloat16,))
    _check_cuda("forward_dropout", q, k, v)
    B, Hq, Hkv, Nq, Nk, d = _shape(q, k)
    scale = d ** -0.5 if scale is None else float(scale)
    o = torch.empty_like(q)
    L = torch.empty(B, Hq, Nq, device=q.device, dtype=torch.float32)
    with _on(q):
        _check(fa_fwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              L.data_ptr(), B, Hq, Hkv, Nq, Nk, d, scale, causal, p_drop, seed,
                              offset, _stream(q)), "fa_fwd_dropout")
    return o, L


def backward_dropout(q, k, v, o, lse, dout, p_drop, seed, offset=0, scale=None, causal=False,
                     workspace=None):
    """dQ, dK, dV of forward_dropout with the same seed and offset."""
    import torch
    _check_qkv("backward_dropout", q, k, v, (torch.bfloat16,))
    _check_bwd_in("backward_dropout", q, o, lse, dout)
    _check_cuda("backward_dropout", q, k, v, o, lse, dout)
    B, Hq, Hkv, Nq, Nk, d = _shape(q, k)
    scale = d ** -0.5 if scale is None else float(scale)
    workspace = _workspace("backward_dropout", workspace, B, Hq, Nq, d, q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    with _on(q):
        _check(fa_bwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                              dv.data_ptr(), workspace.data_ptr(), B, Hq, Hkv, Nq, Nk, d, scale,
                              causal, p_drop, seed, offset, _stream(q)), "fa_bwd_dropout")
    return dq, dk, dv


def backward(q, k, v, o, lse, dout, scale=None, causal=False, workspace=None):
    """dQ, dK, dV for f = sum(O * dout); o and lse from ``forward``."""
    import torch
    _check_qkv("backward", q, k, v, (torch.bfloat16, torch.float32))
    _check_bwd_in("backward", q, o, lse, dout)
    _check_cuda("backward", q, k, v, o, lse, dout)
    B, Hq, Hkv, Nq, Nk, d = _shape(q, k)
    scale = d ** -0.5 if scale is None else float(scale)
    workspace = _workspace("backward", workspace, B, Hq, Nq, d, q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    fn = fa_bwd if q.dtype == torch.bfloat16 else fa_bwd_f32
    with _on(q):
        _check(fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                  dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                  workspace.data_ptr(), B, Hq, Hkv, Nq, Nk, d, scale, causal, _stream(q)),
               fn.__name__)
    return dq, dk, dv
