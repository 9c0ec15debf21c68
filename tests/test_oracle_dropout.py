"""Pins for the dropout part of the float64 oracle (CPU only): the Philox4x32-10
generator against its published known-answer vectors, the keep-mask
statistics, p = 0 reducing to plain attention, central finite differences of
the dropout forward (the mask is a fixed function of the seed, so the output
is smooth in Q, K, V), the expectation over masks, and the row forms.  Planted
mistakes in the dropout formulas must each fail at least one pin."""
import types

import numpy as np
import pytest

import oracle.attention as OA

RNG = np.random.default_rng(4321)


def rnd(*shape):
    return RNG.standard_normal(shape)


def impl_real():
    return types.SimpleNamespace(fwd=OA.dropout_forward, bwd=OA.dropout_backward,
                                 keep=OA.dropout_keep)


def test_philox_known_answers():
    """Known-answer vectors of Philox4x32-10 distributed with the generator
    (Random123, accompanying Salmon et al., SC 2011)."""
    cases = [((0, 0, 0, 0), (0, 0), (0x6627e8d5, 0xe169c58d, 0xbc57ac4c, 0x9b00dbd8)),
             ((0xffffffff,) * 4, (0xffffffff,) * 2, (0x408f276d, 0x41c83b0e, 0xa20bc7c6, 0x6d5451fd)),
             ((0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344), (0xa4093822, 0x299f31d0),
              (0xd16cfe09, 0x94fdcceb, 0x5001e420, 0x24126ea1))]
    for ctr, key, want in cases:
        got = OA.philox4x32_10(*ctr, *key)
        assert tuple(int(x) for x in got) == want


def pin_mask_statistics(impl):
    """p = 0 keeps everything; the kept fraction is 1 - p within 5 sigma;
    heads, offsets and seeds give (nearly) independent masks."""
    rows, cols = np.arange(200), np.arange(400)
    assert impl.keep(0, rows, cols, 0.0, 5, 0).all()
    n = rows.size * cols.size
    for p in (0.1, 0.5, 0.9):
        z = impl.keep(7, rows, cols, p, 99, 3)
        assert abs(z.mean() - (1 - p)) <= 5 * np.sqrt(p * (1 - p) / n)
        for other in (impl.keep(8, rows, cols, p, 99, 3), impl.keep(7, rows, cols, p, 99, 4),
                      impl.keep(7, rows, cols, p, 100, 3)):
            agree = (z == other).mean()
            expect = p * p + (1 - p) * (1 - p)
            assert abs(agree - expect) <= 5 * np.sqrt(expect * (1 - expect) / n)


def pin_p_zero(impl):
    """p = 0 is plain attention, forward and backward."""
    q, k, v, do = rnd(1, 2, 7, 4), rnd(1, 1, 7, 4), rnd(1, 1, 7, 4), rnd(1, 2, 7, 4)
    for causal in (False, True):
        o, l = impl.fwd(q, k, v, 0.6, causal, 0.0, 11, 0)
        o0, l0 = OA.forward(q, k, v, 0.6, causal)
        np.testing.assert_allclose(o, o0, atol=1e-14)
        np.testing.assert_allclose(l, l0, atol=1e-14)
        for a, b in zip(impl.bwd(q, k, v, do, 0.6, causal, 0.0, 11, 0),
                        OA.backward(q, k, v, do, 0.6, causal)):
            np.testing.assert_allclose(a, b, atol=1e-13)


def pin_finite_differences(impl):
    """Central differences of f = sum(O * dO) (fixed mask) match the gradients."""
    h = 1e-6
    for causal, (hq, hkv) in ((False, (2, 1)), (True, (2, 2)), (True, (1, 1))):
        n, d = 9, 5
        q, k, v, do = rnd(1, hq, n, d), rnd(1, hkv, n, d), rnd(1, hkv, n, d), rnd(1, hq, n, d)
        args = (0.7, causal, 0.35, 2024, 5)
        dq, dk, dv, _ = impl.bwd(q, k, v, do, *args)

        def f(q_, k_, v_):
            return float(np.sum(impl.fwd(q_, k_, v_, *args)[0] * do))
        for x, g, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
            num = np.zeros_like(x)
            it = np.nditer(x, flags=["multi_index"])
            for _ in it:
                idx = it.multi_index
                xp, xm = x.copy(), x.copy()
                xp[idx] += h
                xm[idx] -= h
                ins_p = [q, k, v]
                ins_m = [q, k, v]
                ins_p[which], ins_m[which] = xp, xm
                num[idx] = (f(*ins_p) - f(*ins_m)) / (2 * h)
            np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-7)


def pin_expectation(impl):
    """Averaged over masks (offsets), O approaches the undropped O: inverted
    dropout is unbiased.  Elementwise within 6 standard errors."""
    q, k, v = rnd(1, 1, 6, 4), rnd(1, 1, 6, 4), rnd(1, 1, 6, 4)
    o0, _ = OA.forward(q, k, v, 0.5, False)
    samples = np.stack([impl.fwd(q, k, v, 0.5, False, 0.4, 77, off)[0] for off in range(600)])
    mean, se = samples.mean(axis=0), samples.std(axis=0) / np.sqrt(len(samples))
    assert np.all(np.abs(mean - o0) <= 6 * se + 1e-12)


def pin_d_identity(impl):
    """D = rowsum(P * dP) equals rowsum(dO * O) with dropout too."""
    q, k, v, do = rnd(2, 2, 8, 4), rnd(2, 1, 8, 4), rnd(2, 1, 8, 4), rnd(2, 2, 8, 4)
    o, _ = impl.fwd(q, k, v, 0.5, True, 0.25, 3, 9)
    _, _, _, D = impl.bwd(q, k, v, do, 0.5, True, 0.25, 3, 9)
    np.testing.assert_allclose(D, np.sum(do * o, axis=-1), atol=1e-12)


def pin_row_forms(impl):
    """Row-subset forms equal the full forms (used at full workload sizes)."""
    B, Hq, Hkv, n, d = 1, 4, 2, 37, 6
    q, k, v, do = rnd(B, Hq, n, d), rnd(B, Hkv, n, d), rnd(B, Hkv, n, d), rnd(B, Hq, n, d)
    args = (0.45, True, 0.3, 555, 2)
    o, lse = impl.fwd(q, k, v, *args)
    dq, dk, dv, D = impl.bwd(q, k, v, do, *args)
    rows = np.array([0, 5, 17, 36])
    for h in range(Hq):
        kh = h // 2
        orow, lrow = OA.dropout_forward_rows(q[0, h], k[0, kh], v[0, kh], 0.45, True, rows, h,
                                             0.3, 555, 2)
        np.testing.assert_allclose(orow, o[0, h, rows], atol=1e-13)
        np.testing.assert_allclose(lrow, lse[0, h, rows], atol=1e-13)
        dqr, Dr = OA.dropout_backward_rows(q[0, h], k[0, kh], v[0, kh], do[0, h], 0.45, True, rows,
                                           h, 0.3, 555, 2)
        np.testing.assert_allclose(dqr, dq[0, h, rows], atol=1e-12)
        np.testing.assert_allclose(Dr, D[0, h, rows], atol=1e-12)
    kv_rows = np.array([0, 13, 36])
    for kh in range(Hkv):
        dkr, dvr = OA.dropout_backward_kv_rows([q[0, 2 * kh], q[0, 2 * kh + 1]], k[0, kh], v[0, kh],
                                               [do[0, 2 * kh], do[0, 2 * kh + 1]],
                                               [2 * kh, 2 * kh + 1], 0.45, True, kv_rows, 0.3, 555,
                                               2, chunk=7)
        np.testing.assert_allclose(dkr, dk[0, kh, kv_rows], atol=1e-12)
        np.testing.assert_allclose(dvr, dv[0, kh, kv_rows], atol=1e-12)


PINS = [pin_mask_statistics, pin_p_zero, pin_finite_differences, pin_expectation, pin_d_identity,
        pin_row_forms]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_dropout_pin(pin):
    pin(impl_real())


def _mutant(name):
    impl = impl_real()
    if name == "no_rescale":
        f = impl.fwd
        impl.fwd = lambda q, k, v, s, c, p, sd, off: (lambda r: (r[0] * (1 - p), r[1]))(
            f(q, k, v, s, c, p, sd, off))
    elif name == "dp_unmasked":
        def bwd(q, k, v, do, scale, causal, p, seed, offset):
            q_, k_, v_, do_ = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
            dq, dk, dv, D = OA.dropout_backward(q_, k_, v_, do_, scale, causal, p, seed, offset)
            B, Hq, Nq, d = q_.shape
            Hkv, Nk = k_.shape[1], k_.shape[2]
            dq2, dk2 = np.zeros_like(q_), np.zeros_like(k_)
            for b in range(B):
                for h in range(Hq):
                    kh = h // (Hq // Hkv)
                    pr = OA.probs(q_[b, h], k_[b, kh], scale, causal)
                    dp = (do_[b, h] @ v_[b, kh].T) / (1 - p)        # plant: mask dropped
                    ds = pr * (dp - D[b, h][:, None])
                    dq2[b, h] = scale * ds @ k_[b, kh]
                    dk2[b, kh] += scale * ds.T @ q_[b, h]
            return dq2, dk2, dv, D
        impl.bwd = bwd
    elif name == "mask_shared_by_heads":
        impl.keep = lambda bh, r, c, p, s, o: OA.dropout_keep(0, r, c, p, s, o)
    elif name == "dv_unmasked":
        b = impl.bwd

        def bwd(q, k, v, do, scale, causal, p, seed, offset):
            dq, dk, dv, D = b(q, k, v, do, scale, causal, p, seed, offset)
            pr = OA.probs(np.asarray(q, float)[0, 0], np.asarray(k, float)[0, 0], scale, causal)
            return dq, dk, dv * 0 + (pr.T @ np.asarray(do, float)[0, 0])[None, None] / (1 - p), D
        impl.bwd = bwd
    else:
        raise KeyError(name)
    return impl


@pytest.mark.parametrize("mutant", ["no_rescale", "dp_unmasked", "mask_shared_by_heads",
                                    "dv_unmasked"])
def test_dropout_pins_catch_mutants(mutant):
    impl = _mutant(mutant)
    caught = []
    for pin in PINS:
        try:
            pin(impl)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught {mutant}"
