"""Float64 CPU oracle for the FP8 (e4m3) attention forward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` call it.  It shares no code with the CUDA library.

Source: the "FlashAttention" wiki (newton.com.tw), FlashAttention-3
paragraph, names low-precision FP8 computation as one of the Hopper features
FA3 uses, and gives no further definition.  Readings adopted here:

* Inputs Q, K, V are OCP FP8 E4M3 codes (1 sign bit, 4 exponent bits with
  bias 7, 3 mantissa bits; exponent field 0 is subnormal, m/8 * 2^-6; no
  infinities; S.1111.111 is NaN; largest finite 448), one byte per element,
  each tensor with one float32 dequantisation factor (descale): the tensor
  the user means is descale * decode(code).
* The operation is exact attention of those dequantised tensors:
      O = softmax(scale * (dq Q^)(dk K^)^T [+ causal mask]) (dv V^),
      L = log-sum-exp of the scaled scores (natural log),
  the same definition as the bf16 path (``oracle.attention.forward``).
* The kernel holds the probabilities P in e4m3 for the P V product.  That
  rounding is not part of the definition: it is an error source whose size
  ``p_quantisation_bounds`` gives from e4m3's arithmetic, and the parity
  tests compare against the exact values with those bounds.

Parity: ``e4m3_decode`` is pinned to the OCP E4M3 code table (spec values)
and to torch's float8_e4m3fn conversion for all 256 codes;
``fp8_forward`` to torch's float64 SDPA on the dequantised tensors and to the
scale-folding identities of the definition; ``p_quantisation_bounds`` to a
brute-force online-softmax run that rounds P to e4m3 (tests/test_oracle_fp8.py).
"""
from __future__ import annotations

import numpy as np

from .attention import forward

__all__ = ["e4m3_decode", "e4m3_round", "fp8_forward", "fp8_forward_rows",
           "p_quantisation_bounds", "stored_p_forward", "P_SHIFT_LOG2", "P_RESCALE_LOG2"]

# Reading of the kernel's P storage, fixed by the method's FP8 variant here:
# p is stored as e4m3(2^P_SHIFT_LOG2 * 2^(x - m_run)) where m_run (base-2
# units) is a running row maximum that lags the true one by at most
# P_RESCALE_LOG2, so every stored value is at most 2^(4 + 4) = 256 < 448.
P_SHIFT_LOG2 = 4
P_RESCALE_LOG2 = 4


def e4m3_decode(codes) -> np.ndarray:
    """float64 values of OCP FP8 E4M3 codes (uint8 array-like)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = sign * np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = sign * np.ldexp(m / 8.0, -6)
    out = np.where(e == 0, sub, normal)
    return np.where((e == 0xF) & (m == 0x7), np.nan, out)


def _dequant(codes, descale):
    return e4m3_decode(codes) * float(descale)


def fp8_forward(q8, k8, v8, descale_q, descale_k, descale_v, scale, causal):
    """(O, L) of the dequantised tensors; q8 [B,Hq,N,d], k8/v8 [B,Hkv,N,d]
    uint8 codes."""
    return forward(_dequant(q8, descale_q), _dequant(k8, descale_k), _dequant(v8, descale_v),
                   scale, causal)


def fp8_forward_rows(q8_2, k8_2, v8_2, descale_q, descale_k, descale_v, scale, causal, rows):
    """(O rows, L rows) of one head for the given query rows (2-D code arrays)."""
    from .attention import forward_rows
    return forward_rows(_dequant(q8_2, descale_q), _dequant(k8_2, descale_k),
                        _dequant(v8_2, descale_v), scale, causal, rows)


def p_quantisation_bounds(q2, k2, v2, scale, causal, rows=None):
    """Error bounds on O from holding P in e4m3, for one head (float64 inputs
    already dequantised).

    With x_j the scaled score in base 2 and m_k the running maximum used when
    key j's block was processed (m_k <= the final running maximum m_f <= the
    true maximum), the stored value is y = e4m3(2^s 2^(x_j - m_k)), s =
    P_SHIFT_LOG2.  Round to nearest in e4m3 errs by at most 2^-4 y for normal
    y (>= 2^-6) and by at most 2^-10 below (half the subnormal spacing 2^-9).
    Brought to the final units (times 2^(m_k - m_f) <= 1, over 2^s) and
    divided by the row sum l_f = sum_j 2^(x_j - m_f) >= l = sum_j
    exp(s_j - max s) >= 1, the weight w_j = p_j / l errs by at most
        e_j = max(2^-4 w_j, 2^-(10 + s) / l).
    Returns (elementwise, rms):
      elementwise[i, c] = sum_j e_ij |v_jc|        (worst case)
      rms = sqrt(sum_ijc kappa_ij^2 v_jc^2)         (independent rounding)
    with kappa_ij = max(0.0266 w_ij, 2^-(10 + s) / (sqrt(3) l_i)): 0.0266 is
    the root-mean-square relative error of round to nearest with 3 mantissa
    bits for values spread evenly in log scale,
    sqrt(2^-6 / 12 * (3/8) / ln 2)."""
    from .attention import _row_chunk_scores, scores
    if rows is None:
        s = scores(q2, k2, scale, causal)
    else:
        s = _row_chunk_scores(q2, k2, scale, causal, np.asarray(rows))
    mx = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - mx)
    l = np.sum(e, axis=1, keepdims=True)
    w = e / l
    v2 = np.asarray(v2, dtype=np.float64)
    floor_abs = 2.0 ** -(10 + P_SHIFT_LOG2) / l
    e_max = np.maximum(2.0 ** -4 * w, floor_abs)
    e_max = np.where(w > 0, e_max, 0.0)          # masked keys are never stored
    elementwise = e_max @ np.abs(v2)
    kappa_rel = np.sqrt(2.0 ** -6 / 12.0 * 0.375 / np.log(2.0))
    kappa = np.maximum(kappa_rel * w, floor_abs / np.sqrt(3.0))
    kappa = np.where(w > 0, kappa, 0.0)
    rms = float(np.sqrt(np.sum((kappa ** 2) @ (v2 ** 2))))
    return elementwise, rms


def e4m3_round(y) -> np.ndarray:
    """Round non-negative float64 values to the nearest OCP E4M3 value, ties
    to even, saturating at the largest finite value 448 (the satfinite
    conversion).  Subnormals: multiples of 2^-9 below 2^-6; normals: 3
    mantissa bits, a step of 2^(e-3) in [2^e, 2^(e+1))."""
    y = np.asarray(y, dtype=np.float64)
    if np.any(y < 0) or np.any(np.isnan(y)):
        raise ValueError("e4m3_round takes non-negative values")
    out = np.empty_like(y)
    sub = y < 2.0 ** -6
    out[sub] = np.rint(y[sub] / 2.0 ** -9) * 2.0 ** -9
    nz = ~sub
    e = np.floor(np.log2(np.where(nz, y, 1.0)))
    step = np.exp2(e - 3)
    out[nz] = (np.rint(y / step) * step)[nz]
    return np.minimum(out, 448.0)


def stored_p_forward(x2, v2, shift=P_SHIFT_LOG2, tau=P_RESCALE_LOG2, block=128, group=32):
    """O of one head when P is held as the kernel's reading above holds it:
    the online softmax with deferred normalisation (blog section 4.1) in
    float64 over key blocks of `block`, each stored value rounded by
    ``e4m3_round``: y = e4m3(2^shift 2^(x - m)), the row sum over the
    unrounded values, and the running maximum m (base 2) refreshed only when
    some row of a `group` of consecutive rows grows by more than `tau` (the
    first block always sets it).  x2: scaled scores in base 2, [n, nk], -inf
    where masked; v2: [nk, d] float64.  This models the error source that
    ``p_quantisation_bounds`` bounds; it is not the definition of O."""
    x2 = np.asarray(x2, dtype=np.float64)
    v2 = np.asarray(v2, dtype=np.float64)
    n, nk = x2.shape
    m = np.full(n, -np.inf)
    l = np.zeros(n)
    acc = np.zeros((n, v2.shape[1]))
    for j0 in range(0, nk, block):
        x = x2[:, j0:j0 + block]
        m_new = np.maximum(m, x.max(axis=1))
        for g0 in range(0, n, group):
            sl = slice(g0, g0 + group)
            if j0 == 0 or np.any(m_new[sl] - m[sl] > tau):
                alpha = np.where(np.isfinite(m[sl]), np.exp2(m[sl] - m_new[sl]), 0.0)
                acc[sl] *= alpha[:, None]
                l[sl] *= alpha
                m[sl] = m_new[sl]
        mu = np.where(np.isfinite(m), m, 0.0)
        y = np.exp2(x - mu[:, None] + shift)
        l += y.sum(axis=1)
        acc += e4m3_round(y) @ v2[j0:j0 + block]
    return acc / l[:, None]

