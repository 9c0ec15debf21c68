"""Shared helpers of the GPU parity tests: run the library on seeded inputs,
run the float64 oracle on the same bits, and compare with the tolerances of
the method's precision.

Tolerances:
* bf16 inputs, f32 accumulation: O is stored in bf16 (round to nearest
  even), whose half-ulp alone reaches 0.0039-0.0078 for |O| in [1, 4), above
  the 6e-3 error budget; the check is, element by element,
  |O - O_ref| <= 6e-3 + ulp_bf16(O_ref) / 2, i.e. 6e-3 on top of the output
  rounding.  L (f32): max |L - L_ref| <= 1e-3.  dQ, dK, dV: relative
  Frobenius error <= 1.5e-2.
* float32 inputs: max abs error <= 1e-4 on O, L, dQ, dK, dV.
"""
from __future__ import annotations

import numpy as np
import torch

import attn_inputs
import exact_io_aware_50_b200 as F
import oracle

O_TOL_BF16 = 6e-3
L_TOL = 1e-3
GRAD_REL_TOL = 1.5e-2
F32_TOL = 1e-4


def to_dev(x):
    return {k: v.cuda() for k, v in x.items()}


def bf16_round(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(a).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()


def half_ulp_bf16(a: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers at |a| (8 significant bits)."""
    mag = np.maximum(np.abs(a), 2.0 ** -126)
    return np.ldexp(1.0, np.floor(np.log2(mag)).astype(np.int64) - 8)


def check_o(o_gpu: np.ndarray, o_ref: np.ndarray, dtype: str, what="O"):
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite values"
    if dtype == "bf16":
        raw = np.abs(o_gpu - o_ref)
        excess = raw - half_ulp_bf16(o_ref)
        i = np.unravel_index(np.argmax(excess), excess.shape)
        err = float(excess[i])
        assert err <= O_TOL_BF16, (f"{what}: |O - O_ref| - ulp/2 = {err:.3g} > {O_TOL_BF16} at {i} "
                                   f"(gpu {o_gpu[i]:.6g}, ref {o_ref[i]:.6g}, raw max {raw.max():.3g})")
    else:
        err = np.max(np.abs(o_gpu - o_ref))
        assert err <= F32_TOL, f"{what}: max abs err {err:.3g} > {F32_TOL}"
    return err


def check_l(l_gpu, l_ref, dtype):
    assert np.isfinite(l_gpu).all()
    err = np.max(np.abs(l_gpu - l_ref))
    tol = L_TOL if dtype == "bf16" else F32_TOL
    assert err <= tol, f"L: max abs err {err:.3g} > {tol}"
    return err


def check_grad(g_gpu, g_ref, dtype, what):
    assert np.isfinite(g_gpu).all(), f"{what}: non-finite values"
    if dtype == "bf16":
        ref_norm = np.linalg.norm(g_ref)
        if ref_norm == 0.0:
            # exact zero gradient (e.g. a single key): only rounding noise allowed
            err = np.max(np.abs(g_gpu))
            assert err <= 1e-4, f"{what}: reference is zero, max |gpu| = {err:.3g}"
            return err
        rel = np.linalg.norm(g_gpu - g_ref) / ref_norm
        assert rel <= GRAD_REL_TOL, f"{what}: relative Frobenius error {rel:.3g} > {GRAD_REL_TOL}"
        return rel
    err = np.max(np.abs(g_gpu - g_ref))
    assert err <= F32_TOL, f"{what}: max abs err {err:.3g} > {F32_TOL}"
    return err


def f64(t):
    return attn_inputs.as_f64(t)


def run_full_check(B, Hq, Hkv, Nq, Nk, d, causal, dtype="bf16", seed=0, q_mul=1.0, k_add=0.0,
                   backward=True, scale=None, cta_pair=False):
    """Whole-tensor parity of forward (and backward) against the oracle."""
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    x = attn_inputs.draw(B, Hq, Hkv, Nq, Nk, d, seed, dt, q_mul, k_add)
    scale = d ** -0.5 if scale is None else scale
    g = to_dev(x)
    o, lse = F.forward(g["q"], g["k"], g["v"], scale, causal, cta_pair=cta_pair)
    torch.cuda.synchronize()
    assert F.fa_device_status() == F.FA_OK
    q, k, v, do = (f64(x[n]) for n in ("q", "k", "v", "do"))
    o_ref, l_ref = oracle.forward(q, k, v, scale, causal)
    check_o(f64(o), o_ref, dtype)
    check_l(f64(lse), l_ref, dtype)
    if not backward:
        return
    dq, dk, dv = F.backward(g["q"], g["k"], g["v"], o, lse, g["do"], scale, causal)
    torch.cuda.synchronize()
    assert F.fa_device_status() == F.FA_OK
    dq_r, dk_r, dv_r, _ = oracle.backward(q, k, v, do, scale, causal)
    check_grad(f64(dq), dq_r, dtype, "dQ")
    check_grad(f64(dk), dk_r, dtype, "dK")
    check_grad(f64(dv), dv_r, dtype, "dV")
