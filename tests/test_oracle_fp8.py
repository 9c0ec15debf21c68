"""Pins for the FP8 (E4M3) part of the float64 oracle (CPU only).

* ``e4m3_decode`` against the E4M3 values fixed by the OCP 8-bit floating
  point specification (OFP8, E4M3 column: bias 7, no infinities, NaN at
  S.1111.111, max normal 448, min normal 2^-6, min subnormal 2^-9) and
  against torch's float8_e4m3fn conversion for all 256 codes.
* ``fp8_forward`` against torch's float64 scaled_dot_product_attention on the
  dequantised tensors, and against the scale-folding identities of the
  definition (the Q and K factors act as a score scale, the V factor scales O).
* ``p_quantisation_bounds`` against a brute-force online softmax that rounds
  the stored probabilities to e4m3 (torch's conversion), with the running
  maximum lagging by up to the rescale threshold as the kernel allows: the
  worst-case bound holds for every element, a bound with half the relative
  term is broken on peaked rows, and the root-mean-square prediction matches
  the simulated error on diffuse rows.
Planted mistakes in the oracle must each fail at least one pin.
"""
import types

import numpy as np
import pytest
import torch

import oracle.attention as OA
import oracle.fp8 as OF

RNG = np.random.default_rng(8642)


def impl_real():
    return types.SimpleNamespace(decode=OF.e4m3_decode, fwd=OF.fp8_forward)


# --------------------------------------------------------------- decode pins
SPEC_VALUES = {
    0x00: 0.0, 0x80: -0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6,
    0x30: 0.5, 0x38: 1.0, 0x39: 1.125, 0x40: 2.0, 0x3F: 1.875, 0x78: 256.0, 0x7E: 448.0,
    0xFE: -448.0, 0xB8: -1.0, 0x81: -(2.0 ** -9),
}


def pin_decode_spec(impl):
    got = impl.decode(np.array(list(SPEC_VALUES), dtype=np.uint8))
    want = np.array(list(SPEC_VALUES.values()))
    assert np.array_equal(got, want)
    assert np.array_equal(np.signbit(got), np.signbit(want))
    nan = impl.decode(np.array([0x7F, 0xFF], dtype=np.uint8))
    assert np.all(np.isnan(nan))


def pin_decode_library(impl):
    codes = np.arange(256, dtype=np.uint8)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = impl.decode(codes)
    both_nan = np.isnan(got) & np.isnan(want)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    assert np.array_equal(got[~both_nan], want[~both_nan])


# -------------------------------------------------------------- forward pins
def _codes(shape, spread=1.0):
    x = torch.from_numpy(RNG.standard_normal(shape) * spread).to(torch.float32)
    return x.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def pin_forward_library(impl):
    import torch.nn.functional as F
    for causal in (False, True):
        q8, k8, v8 = _codes((1, 2, 37, 16), 40.0), _codes((1, 2, 37, 16), 40.0), _codes((1, 2, 37, 16), 40.0)
        dq, dk, dv = 0.0125, 0.02, 0.5
        o, L = impl.fwd(q8, k8, v8, dq, dk, dv, 0.25, causal)
        tq = torch.from_numpy(OF.e4m3_decode(q8) * dq)
        tk = torch.from_numpy(OF.e4m3_decode(k8) * dk)
        tv = torch.from_numpy(OF.e4m3_decode(v8) * dv)
        want = F.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=0.25).numpy()
        assert np.allclose(o, want, rtol=1e-10, atol=1e-12)
        s = 0.25 * (tq @ tk.transpose(-1, -2)).numpy()
        if causal:
            s = np.where(np.tril(np.ones((37, 37), dtype=bool)), s, -np.inf)
        m = s.max(-1, keepdims=True)
        assert np.allclose(L, (m + np.log(np.exp(s - m).sum(-1, keepdims=True)))[..., 0], atol=1e-12)


def pin_forward_fold(impl):
    """Q and K factors only multiply the score scale; the V factor scales O."""
    q8, k8, v8 = _codes((2, 2, 50, 32), 30.0), _codes((2, 1, 50, 32), 30.0), _codes((2, 1, 50, 32), 30.0)
    a, b, c = 0.03125, 0.0078125, 3.0
    o1, l1 = impl.fwd(q8, k8, v8, a, b, c, 0.2, True)
    o2, l2 = impl.fwd(q8, k8, v8, 1.0, 1.0, 1.0, 0.2 * a * b, True)
    assert np.allclose(o1, o2 * c, rtol=1e-10, atol=1e-12)
    assert np.allclose(l1, l2, atol=1e-12)


PINS = [pin_decode_spec, pin_decode_library, pin_forward_library, pin_forward_fold]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_fp8_pin(pin):
    pin(impl_real())


def _mutant(name):
    real = impl_real()

    def decode_bias8(c):
        c = np.asarray(c, dtype=np.uint8).astype(np.int64)
        e, m = (c >> 3) & 0xF, c & 7
        v = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1 + m / 8.0, e - 8))
        return np.where(c & 0x80, -v, v)

    def decode_sub_as_normal(c):
        c = np.asarray(c, dtype=np.uint8).astype(np.int64)
        e, m = (c >> 3) & 0xF, c & 7
        v = np.ldexp(1 + m / 8.0, e - 7)
        v = np.where((e == 15) & (m == 7), np.nan, v)
        return np.where(c & 0x80, -v, v)

    def fwd_no_dv(q8, k8, v8, dq, dk, dv, scale, causal):
        return OF.fp8_forward(q8, k8, v8, dq, dk, 1.0, scale, causal)

    def fwd_dq_twice(q8, k8, v8, dq, dk, dv, scale, causal):
        return OF.fp8_forward(q8, k8, v8, dq * dq, dk, dv, scale, causal)

    def fwd_dk_as_dv(q8, k8, v8, dq, dk, dv, scale, causal):
        return OF.fp8_forward(q8, k8, v8, dq, dv, dv, scale, causal)

    table = {"decode_bias8": dict(decode=decode_bias8),
             "decode_subnormal_as_normal": dict(decode=decode_sub_as_normal),
             "descale_v_dropped": dict(fwd=fwd_no_dv),
             "descale_q_twice": dict(fwd=fwd_dq_twice),
             "descale_k_swapped": dict(fwd=fwd_dk_as_dv)}
    return types.SimpleNamespace(**{**vars(real), **table[name]})


@pytest.mark.parametrize("mutant", ["decode_bias8", "decode_subnormal_as_normal",
                                    "descale_v_dropped", "descale_q_twice",
                                    "descale_k_swapped"])
def test_fp8_pins_catch_mutants(mutant):
    impl = _mutant(mutant)
    caught = False
    for pin in PINS:
        try:
            pin(impl)
        except AssertionError:
            caught = True
    assert caught, f"no pin caught {mutant}"


# ------------------------------------------------- P quantisation bound pins
def _e4m3_round(y):
    return torch.from_numpy(y).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def quantised_online(q, k, v, scale, causal, block=128, group=32, shift=OF.P_SHIFT_LOG2,
                     tau=OF.P_RESCALE_LOG2):
    """Online softmax with deferred normalisation in float64 whose stored
    probabilities are rounded to e4m3: y = e4m3(2^shift 2^(x - m)), the row
    sum over the unrounded values, and the running maximum m refreshed only
    when some row of a ``group`` grows by more than ``tau`` (base 2)."""
    n, nk = q.shape[0], k.shape[0]
    x_all = OA.scores(q, k, scale, causal) / np.log(2.0)
    m = np.full(n, -np.inf)
    l = np.zeros(n)
    acc = np.zeros((n, v.shape[1]))
    for j0 in range(0, nk, block):
        x = x_all[:, j0:j0 + block]
        m_new = np.maximum(m, x.max(axis=1))
        first = j0 == 0
        for g0 in range(0, n, group):
            sl = slice(g0, g0 + group)
            grow = m_new[sl] - m[sl]
            if first or np.any(grow > tau):
                alpha = np.where(np.isfinite(m[sl]), np.exp2(m[sl] - m_new[sl]), 0.0)
                acc[sl] *= alpha[:, None]
                l[sl] *= alpha
                m[sl] = m_new[sl]
        mu = np.where(np.isfinite(m), m, 0.0)
        y = np.exp2(x - mu[:, None] + shift)
        assert y.max() <= 256.0 + 1e-9
        l += y.sum(axis=1)
        acc += _e4m3_round(y) @ v[j0:j0 + block]
    return acc / l[:, None]


@pytest.mark.parametrize("case", ["diffuse", "peaked", "causal_peaked", "adversarial"])
def test_p_quantisation_worst_case_bound(case):
    n, d = 384, 64
    spread = {"diffuse": 1.0, "peaked": 6.0, "causal_peaked": 6.0, "adversarial": 3.0}[case]
    causal = case.startswith("causal")
    q = RNG.standard_normal((n, d)) * spread
    k = RNG.standard_normal((n, d))
    if case == "adversarial":
        # scores that grow along the keys: the running max keeps lagging
        k = k + np.linspace(0, 4, n)[:, None] * np.sign(q.mean(0))[None, :]
    v = RNG.standard_normal((n, d))
    scale = d ** -0.5
    o_exact, _ = OA.forward(q[None, None], k[None, None], v[None, None], scale, causal)
    o_sim = quantised_online(q, k, v, scale, causal)
    bound, _ = OF.p_quantisation_bounds(q, k, v, scale, causal)
    err = np.abs(o_sim - o_exact[0, 0])
    assert np.all(err <= bound * (1 + 1e-9) + 1e-15)
    if case != "diffuse":
        # half the relative term is not a bound: the 2^-4 is needed
        w = OA.probs(q, k, scale, causal)
        tighter = (0.5 * 2.0 ** -4 * w) @ np.abs(v)
        assert np.any(err > tighter)


def test_p_quantisation_rms_prediction():
    ratios = []
    for h in range(4):
        n, d = 512, 64
        q = RNG.standard_normal((n, d))
        k = RNG.standard_normal((n, d))
        v = RNG.standard_normal((n, d))
        scale = d ** -0.5
        o_exact, _ = OA.forward(q[None, None], k[None, None], v[None, None], scale, h % 2 == 1)
        o_sim = quantised_online(q, k, v, scale, h % 2 == 1)
        _, rms = OF.p_quantisation_bounds(q, k, v, scale, h % 2 == 1)
        ratios.append(np.sqrt(np.sum((o_sim - o_exact[0, 0]) ** 2)) / rms)
    # the model slightly over-predicts rows dominated by their maximum (stored
    # exactly as 2^4): causal heads land near 0.75, full ones near 0.95
    assert all(0.5 < r < 1.25 for r in ratios), ratios


def test_p_quantisation_rows_form():
    n, d = 300, 32
    q, k, v = (RNG.standard_normal((n, d)) for _ in range(3))
    full, _ = OF.p_quantisation_bounds(q, k, v, 0.3, True)
    rows = np.array([0, 7, 128, 299])
    part, _ = OF.p_quantisation_bounds(q, k, v, 0.3, True, rows=rows)
    assert np.allclose(part, full[rows], rtol=1e-12, atol=1e-15)


def test_fp8_forward_rows_matches_full():
    q8, k8, v8 = _codes((1, 1, 200, 32), 50.0), _codes((1, 1, 200, 32), 50.0), _codes((1, 1, 200, 32), 50.0)
    o, L = OF.fp8_forward(q8, k8, v8, 0.01, 0.02, 0.5, 0.2, True)
    rows = np.array([0, 1, 99, 199])
    orow, lrow = OF.fp8_forward_rows(q8[0, 0], k8[0, 0], v8[0, 0], 0.01, 0.02, 0.5, 0.2, True, rows)
    assert np.allclose(orow, o[0, 0, rows], rtol=1e-12, atol=1e-14)
    assert np.allclose(lrow, L[0, 0, rows], atol=1e-12)


def test_draw_fp8_inputs():
    """The seeded E4M3 inputs: no NaN codes, factors exact in float32, the
    dequantised tensor within e4m3 rounding of the float32 draw, and the same
    bits on every call."""
    import attn_inputs
    x = attn_inputs.draw_fp8(1, 2, 1, 64, 128, seed=11)
    y = attn_inputs.draw_fp8(1, 2, 1, 64, 128, seed=11)
    raw = attn_inputs.draw(1, 2, 1, 64, 64, 128, 11, torch.float32)
    for n in ("q", "k", "v"):
        codes = x[n].numpy()
        assert codes.dtype == np.uint8
        assert not np.any((codes & 0x7F) == 0x7F)
        ds = x["descale_" + n]
        assert float(np.float32(ds)) == ds
        deq = OF.e4m3_decode(codes) * ds
        ref = raw[n].double().numpy()
        # round to nearest at 3 mantissa bits: relative 2^-4 for normals, 2^-10 * ds below 2^-6 * ds
        assert np.all(np.abs(deq - ref) <= np.maximum(2.0 ** -4 * np.abs(ref), 2.0 ** -10 * ds) * (1 + 1e-6))
        assert np.isclose(np.abs(deq).max(), 448 * ds, rtol=2.0 ** -4)
        assert np.array_equal(codes, y[n].numpy()) and ds == y["descale_" + n]


# ------------------------------------------- stored-P model of the kernel
def test_e4m3_round_grid_midpoints_and_saturation():
    """e4m3_round: every finite non-negative E4M3 value is a fixed point;
    midpoints between neighbours round as torch's float8_e4m3fn conversion
    (round to nearest even); values above 448 saturate (satfinite)."""
    vals = OF.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    assert np.array_equal(OF.e4m3_round(vals), vals)
    mid = (vals[1:] + vals[:-1]) / 2
    assert np.array_equal(OF.e4m3_round(mid), _e4m3_round(mid))
    r = RNG.uniform(0, 448, 20000) * np.exp2(RNG.integers(-14, 1, 20000))
    assert np.array_equal(OF.e4m3_round(r), _e4m3_round(r))
    assert np.all(OF.e4m3_round(np.array([448.0, 460.0, 480.0, 1e9])) == 448.0)


def test_stored_p_forward_matches_simulation_with_library_rounding():
    """stored_p_forward equals quantised_online above (scores from the
    oracle's definition, rounding by torch's e4m3 conversion)."""
    n, d = 300, 64
    q = RNG.standard_normal((n, d)) * 3.0
    k = RNG.standard_normal((n, d))
    v = RNG.standard_normal((n, d))
    scale = d ** -0.5
    for causal in (False, True):
        x2 = OA.scores(q, k, scale, causal) / np.log(2.0)
        a = OF.stored_p_forward(x2, v)
        b = quantised_online(q, k, v, scale, causal)
        assert np.max(np.abs(a - b)) <= 1e-12


def test_stored_p_forward_is_exact_on_the_grid():
    """When every stored value lands on the e4m3 grid (integer base-2 scores
    close to the row maximum), the model reproduces softmax(x) V exactly,
    whichever running maximum it used: a closed form for its recurrence."""
    n, nk, d = 64, 384, 16
    x2 = RNG.integers(-9 - OF.P_SHIFT_LOG2, 1, (n, nk)).astype(np.float64)
    x2[:, 200] += 4      # a growth of exactly tau: no rescale, stored 2^8
    v = RNG.standard_normal((nk, d))
    w = np.exp2(x2 - x2.max(axis=1, keepdims=True))
    exact = (w / w.sum(axis=1, keepdims=True)) @ v
    assert np.max(np.abs(OF.stored_p_forward(x2, v) - exact)) <= 1e-12
