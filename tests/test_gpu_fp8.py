"""GPU parity of the E4M3 forward (fa_fwd_fp8) against the float64 oracle.

The oracle gives the exact attention of the dequantised tensors; the kernel
rounds P to e4m3 for the P V product.  Each element of O must lie within the
worst-case effect of that rounding (``oracle.fp8.p_quantisation_bounds``,
times 1.05 for float32 score and accumulation error) plus half a bf16 ulp of
the output; the Frobenius norm of the error must stay within 1.5 times the
root-mean-square prediction of independent rounding (output rounding
included); L within 1e-3.  Small seeded cases span several tiles and ragged
tails; the training shape with e4m3 inputs is checked on sampled rows."""
import numpy as np
import pytest
import torch

import attn_inputs
import exact_io_aware_50_b200 as F
import oracle.fp8 as OF
from parity import L_TOL, f64, half_ulp_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    F.lib()
    yield


def _run(x, causal, scale):
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    o, lse = F.forward_fp8(g["q"], g["k"], g["v"], g["descale_q"], g["descale_k"], g["descale_v"],
                           scale=scale, causal=causal)
    torch.cuda.synchronize()
    assert F.fa_device_status() == F.FA_OK
    return f64(o), f64(lse)


def _check_head(o_gpu, l_gpu, x, b, h, hkv, causal, scale, rows=None):
    """Returns (sum of squared errors, predicted variance) for this head."""
    q2 = OF.e4m3_decode(x["q"][b, h].numpy()) * x["descale_q"]
    k2 = OF.e4m3_decode(x["k"][b, hkv].numpy()) * x["descale_k"]
    v2 = OF.e4m3_decode(x["v"][b, hkv].numpy()) * x["descale_v"]
    if rows is None:
        rows = np.arange(q2.shape[0])
    from oracle.attention import forward_rows
    o_ref, l_ref = forward_rows(q2, k2, v2, scale, causal, rows)
    bound, rms = OF.p_quantisation_bounds(q2, k2, v2, scale, causal, rows=rows)
    og, lg = o_gpu[rows], l_gpu[rows]
    assert np.isfinite(og).all() and np.isfinite(lg).all()
    err = np.abs(og - o_ref)
    allowed = 1.05 * bound + half_ulp_bf16(o_ref) + 1e-6
    i = np.unravel_index(np.argmax(err - allowed), err.shape)
    assert err[i] <= allowed[i], (f"b={b} h={h} row {rows[i[0]]} col {i[1]}: |O - O_ref| = "
                                  f"{err[i]:.3g} > {allowed[i]:.3g} (gpu {og[i]:.6g}, ref {o_ref[i]:.6g})")
    lerr = np.max(np.abs(lg - l_ref))
    assert lerr <= L_TOL, f"b={b} h={h}: max |L - L_ref| = {lerr:.3g}"
    out_var = np.sum((half_ulp_bf16(o_ref) / np.sqrt(3.0)) ** 2)
    return float(np.sum((og - o_ref) ** 2)), rms ** 2 + float(out_var)


CASES = [(1, 2, 1, 300, 128, True), (2, 2, 2, 257, 128, False), (1, 4, 2, 513, 256, True),
         (1, 2, 2, 1000, 256, False), (1, 1, 1, 1, 128, True), (1, 2, 1, 129, 128, False),
         (1, 2, 2, 640, 128, True)]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(str(v) for v in c))
def test_fp8_small(case):
    B, Hq, Hkv, N, d, causal = case
    x = attn_inputs.draw_fp8(B, Hq, Hkv, N, d, seed=700 + N + d)
    scale = d ** -0.5
    o, lse = _run(x, causal, scale)
    sse = var = 0.0
    for b in range(B):
        for h in range(Hq):
            e, v = _check_head(o[b, h], lse[b, h], x, b, h, h // (Hq // Hkv), causal, scale)
            sse += e
            var += v
    assert np.sqrt(sse) <= 1.5 * np.sqrt(var) + 1e-6, (np.sqrt(sse), np.sqrt(var))


def test_fp8_peaked_scores():
    """Q scaled by 8: most rows dominated by a few keys, running maximum
    growing across blocks (rescales), P values spread over e4m3's range."""
    B, Hq, Hkv, N, d = 1, 2, 2, 777, 128
    x = attn_inputs.draw_fp8(B, Hq, Hkv, N, d, seed=771, q_mul=8.0)
    scale = d ** -0.5
    for causal in (True, False):
        o, lse = _run(x, causal, scale)
        for h in range(Hq):
            _check_head(o[0, h], lse[0, h], x, 0, h, h, causal, scale)


def test_fp8_training_shape_sampled():
    """fp8_causal_b4_h16_n4096_d128 at full size; sampled rows of three heads."""
    w = attn_inputs.FP8_CAUSAL
    x = attn_inputs.make_fp8(w)
    o, lse = _run(x, w.causal, w.scale)
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 2047, 4095],
                                     rng.integers(0, w.N, 18)]))
    sse = var = 0.0
    for b, h in ((0, 0), (1, 7), (3, 15)):
        e, v = _check_head(o[b, h], lse[b, h], x, b, h, h, w.causal, w.scale, rows=rows)
        sse += e
        var += v
    assert np.sqrt(sse) <= 1.5 * np.sqrt(var) + 1e-6, (np.sqrt(sse), np.sqrt(var))


def test_fp8_descale_fold():
    """The same codes with descale_v doubled give exactly twice the bf16
    output (a power of two), and a Q factor doubled against a halved scale
    gives the same O and L bit for bit."""
    x = attn_inputs.draw_fp8(1, 2, 2, 384, 128, seed=9)
    o1, l1 = _run(x, True, 0.1)
    y = dict(x)
    y["descale_v"] = 2.0 * x["descale_v"]
    o2, l2 = _run(y, True, 0.1)
    assert np.array_equal(o2, 2.0 * o1)
    assert np.array_equal(l2, l1)
    z = dict(x)
    z["descale_q"] = 2.0 * x["descale_q"]
    o3, l3 = _run(z, True, 0.05)
    assert np.array_equal(o3, o1) and np.array_equal(l3, l1)


def _e4m3_code(x):
    """Code of an exactly representable E4M3 value."""
    c = torch.tensor([x], dtype=torch.float64).to(torch.float8_e4m3fn).view(torch.uint8).item()
    assert OF.e4m3_decode(np.array([c], np.uint8))[0] == x, x
    return c


def test_fp8_p_storage_matches_the_bound_model():
    """The kernel's P storage is what oracle.fp8's error model assumes:
    e4m3(2^P_SHIFT_LOG2 2^(x - m)) with a running maximum that lags by at most
    P_RESCALE_LOG2.  Every query row is q = (1, 1/2, 0, ...) and each key's
    first two components set its score (scale = ln 2, so scores are in base
    2); probe keys sit where the stored value lands clearly on or off the
    e4m3 subnormal grid, next to block maxima that grow by exactly 4 and then
    by 9.  The kernel's O must equal stored_p_forward's within one bf16 ulp,
    and the model with shift 3 or 5, or threshold 3 or 9, must give an O that
    differs by many ulps, so a change on either side fails this test."""
    N, d = 384, 128
    # base-2 scores, value columns: (key, score, column of its value 256, or
    # column 0 with value 1 for the block maxima)
    probes = [(0, 0.0, 0), (1, -13.5, 1), (2, -13.0, 2),        # block 0, max 0
              (128, 4.0, 0), (129, -10.5, 3),                   # block 1, max grows by 4
              (256, 9.0, 0), (257, -4.5, 4)]                    # block 2, max grows by 9
    a = np.full(N, -448.0)
    vcol = {}
    for key, score, col in probes:
        a[key] = score
        vcol[key] = col
    k = np.zeros((N, d))
    k[:, 0] = np.ceil(a)                 # representable integers for these scores
    k[:, 1] = 2.0 * (a - np.ceil(a))     # 0 or -1, so that a = k0 + k1 / 2
    v = np.zeros((N, d))
    for key, col in vcol.items():
        v[key, col] = 1.0 if col == 0 else 256.0
    q = np.zeros((N, d))
    q[:, 0], q[:, 1] = 1.0, 0.5
    assert np.array_equal(q @ k.T, np.tile(a, (N, 1)))
    enc = np.vectorize(_e4m3_code)
    codes = {n: torch.from_numpy(enc(t).astype(np.uint8)).reshape(1, 1, N, d)
             for n, t in (("q", q), ("k", k), ("v", v))}
    scale = float(np.float32(np.log(2.0)))
    o, lse = F.forward_fp8(codes["q"].cuda(), codes["k"].cuda(), codes["v"].cuda(), 1.0, 1.0, 1.0,
                           scale=scale, causal=False)
    torch.cuda.synchronize()
    assert F.fa_device_status() == F.FA_OK
    o = f64(o)[0, 0]
    x2 = np.tile(a, (N, 1))

    def model(shift, tau):
        return OF.stored_p_forward(x2, v, shift=shift, tau=tau)

    ref = model(OF.P_SHIFT_LOG2, OF.P_RESCALE_LOG2)
    ulp = 2.0 * half_ulp_bf16(ref)
    assert np.all(np.abs(o - ref) <= ulp), np.max(np.abs(o - ref) / ulp)
    for shift, tau in ((3, 4), (5, 4), (4, 3), (4, 9)):
        alt = model(shift, tau)
        assert np.max(np.abs(alt - ref) / ulp) > 8, (shift, tau)
