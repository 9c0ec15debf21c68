"""Pins for the float64 oracle: closed forms, invariants, finite differences,
a library cross-check and the CSDN tutorial's own worked setup.  CPU only.

Each check is written as a function of an oracle "implementation" so the same
checks can be run against planted mistakes (``test_pins_catch_mutants``): a
plausible error anywhere in the oracle must fail at least one pin.
"""
import json
import math
import os
import types

import numpy as np
import pytest
import torch

import oracle.attention as OA

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def real_impl():
    return types.SimpleNamespace(forward=OA.forward, backward=OA.backward, probs=OA.probs,
                                 forward_rows=OA.forward_rows, backward_rows=OA.backward_rows,
                                 backward_kv_rows=OA.backward_kv_rows, lse_rows=OA.lse_rows,
                                 merge_partials=lambda o, l: OA.merge_partials(o, l),
                                 splitkv_forward=lambda *a, **kw: OA.splitkv_forward(*a, **kw))


def rnd(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


# ---------------------------------------------------------------------------
# individual pins; each returns None or raises AssertionError
# ---------------------------------------------------------------------------

def pin_probs_rows(impl):
    """Softmax rows sum to 1, P >= 0, causal P is zero above the diagonal."""
    for causal in (False, True):
        q, k = rnd(13, 5), rnd(13, 5)
        p = impl.probs(q, k, 0.7, causal)
        assert np.all(p >= 0)
        np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-14)
        if causal:
            assert np.all(p[np.triu_indices(13, 1)] == 0)
            assert np.all(np.diag(p) > 0)


def pin_constant_v(impl):
    """Every V row equal to c gives O_i = c; sum_j dV_j = sum_i dO_i."""
    for causal in (False, True):
        q, k, do = rnd(1, 2, 9, 4), rnd(1, 2, 9, 4), rnd(1, 2, 9, 4)
        c = rnd(4)
        v = np.broadcast_to(c, (1, 2, 9, 4)).copy()
        o, _ = impl.forward(q, k, v, 0.5, causal)
        np.testing.assert_allclose(o, np.broadcast_to(c, o.shape), atol=1e-13)
        _, _, dv, _ = impl.backward(q, k, v, do, 0.5, causal)
        np.testing.assert_allclose(dv.sum(axis=2), do.sum(axis=2), atol=1e-12)


def pin_causal_row0(impl):
    """Causal row 0 sees only key 0: O_0 = V_0 and L_0 = scale * q_0 . k_0."""
    q, k, v = rnd(1, 1, 7, 6), rnd(1, 1, 7, 6), rnd(1, 1, 7, 6)
    o, lse = impl.forward(q, k, v, 0.3, True)
    np.testing.assert_allclose(o[0, 0, 0], v[0, 0, 0], atol=1e-14)
    assert abs(lse[0, 0, 0] - 0.3 * float(q[0, 0, 0] @ k[0, 0, 0])) < 1e-13


def pin_zero_q(impl):
    """Q = 0 makes P uniform over the visible keys."""
    k, v = rnd(1, 1, 11, 3), rnd(1, 1, 11, 3)
    q = np.zeros((1, 1, 11, 3))
    o, lse = impl.forward(q, k, v, 0.9, False)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(v[0, 0].mean(axis=0), (11, 3)), atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], math.log(11), atol=1e-14)
    o, lse = impl.forward(q, k, v, 0.9, True)
    prefix = np.cumsum(v[0, 0], axis=0) / np.arange(1, 12)[:, None]
    np.testing.assert_allclose(o[0, 0], prefix, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], np.log(np.arange(1, 12)), atol=1e-14)


def pin_single_key(impl):
    """Nk = 1: O_i = V_0 and dQ = dK = 0 (dS vanishes)."""
    q, k, v, do = rnd(1, 1, 5, 4), rnd(1, 1, 1, 4), rnd(1, 1, 1, 4), rnd(1, 1, 5, 4)
    o, lse = impl.forward(q, k, v, 0.5, False)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(v[0, 0, 0], (5, 4)), atol=1e-15)
    np.testing.assert_allclose(lse[0, 0], 0.5 * (q[0, 0] @ k[0, 0, 0]), atol=1e-14)
    dq, dk, dv, _ = impl.backward(q, k, v, do, 0.5, False)
    assert np.abs(dq).max() < 1e-14 and np.abs(dk).max() < 1e-14
    np.testing.assert_allclose(dv[0, 0, 0], do[0, 0].sum(axis=0), atol=1e-13)


def pin_shift_invariance(impl):
    """Adding c to every K row shifts row i of S by scale*q_i.c: P, O, dQ, dK,
    dV unchanged and L_i shifted by exactly scale*q_i.c."""
    for causal in (False, True):
        q, k, v, do = rnd(1, 2, 8, 4), rnd(1, 2, 8, 4), rnd(1, 2, 8, 4), rnd(1, 2, 8, 4)
        c = rnd(4) * 3
        o1, l1 = impl.forward(q, k, v, 0.4, causal)
        o2, l2 = impl.forward(q, k + c, v, 0.4, causal)
        np.testing.assert_allclose(o2, o1, atol=1e-12)
        np.testing.assert_allclose(l2 - l1, 0.4 * (q @ c), atol=1e-12)
        g1 = impl.backward(q, k, v, do, 0.4, causal)
        g2 = impl.backward(q, k + c, v, do, 0.4, causal)
        for a, b in zip(g1[:3], g2[:3]):
            np.testing.assert_allclose(a, b, atol=1e-11)


def pin_kplus8_bf16(impl):
    """The adversarial +8 shift on bf16-rounded K is exact in float64, so the
    shifted and unshifted problems agree to rounding of the float64 sums."""
    g = torch.Generator().manual_seed(7)
    kb = (torch.randn(1, 1, 16, 8, generator=g) + 8).to(torch.bfloat16).double().numpy()
    q, v = rnd(1, 1, 16, 8), rnd(1, 1, 16, 8)
    o1, l1 = impl.forward(q, kb, v, 8 ** -0.5, True)
    o2, l2 = impl.forward(q, kb - 8.0, v, 8 ** -0.5, True)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1 - l2, 8 ** -0.5 * 8.0 * q.sum(axis=-1), atol=1e-12)


def pin_gradient_identities(impl):
    """rowsum(dS) = 0 => column sums of dK vanish; D = rowsum(dO * O)."""
    for causal in (False, True):
        q, k, v, do = rnd(2, 2, 10, 4), rnd(2, 1, 10, 4), rnd(2, 1, 10, 4), rnd(2, 2, 10, 4)
        dq, dk, dv, D = impl.backward(q, k, v, do, 0.6, causal)
        np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
        o, _ = impl.forward(q, k, v, 0.6, causal)
        np.testing.assert_allclose(D, np.sum(do * o, axis=-1), atol=1e-12)


def pin_permutation(impl):
    """Non-causal O is invariant under a joint permutation of K and V rows."""
    q, k, v = rnd(1, 1, 6, 3), rnd(1, 1, 9, 3), rnd(1, 1, 9, 3)
    perm = RNG.permutation(9)
    o1, l1 = impl.forward(q, k, v, 1.1, False)
    o2, l2 = impl.forward(q, k[:, :, perm], v[:, :, perm], 1.1, False)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(l1, l2, atol=1e-13)


def pin_hand_example(impl):
    """One query, two keys, worked by hand from the definition:
    s = (1, 0) with scale 1, p = (e/(1+e), 1/(1+e)), O = p0 v0 + p1 v1,
    L = ln(1 + e); with dO = (1, 0): dP = (1, 3), D = O_0, dS = p (dP - D)."""
    q = np.array([[[[1.0, 0.0]]]])
    k = np.array([[[[1.0, 0.0], [0.0, 1.0]]]])
    v = np.array([[[[1.0, 2.0], [3.0, 4.0]]]])
    do = np.array([[[[1.0, 0.0]]]])
    e = math.e
    p0, p1 = e / (1 + e), 1 / (1 + e)
    o_exp = [p0 * 1 + p1 * 3, p0 * 2 + p1 * 4]
    o, lse = impl.forward(q, k, v, 1.0, False)
    np.testing.assert_allclose(o[0, 0, 0], o_exp, atol=1e-15)
    assert abs(lse[0, 0, 0] - math.log(1 + e)) < 1e-15
    dq, dk, dv, D = impl.backward(q, k, v, do, 1.0, False)
    Dexp = o_exp[0]
    ds0, ds1 = p0 * (1 - Dexp), p1 * (3 - Dexp)
    np.testing.assert_allclose(dv[0, 0], [[p0, 0.0], [p1, 0.0]], atol=1e-15)
    np.testing.assert_allclose(dq[0, 0, 0], [ds0, ds1], atol=1e-15)
    np.testing.assert_allclose(dk[0, 0], [[ds0, 0.0], [ds1, 0.0]], atol=1e-15)
    assert abs(D[0, 0, 0] - Dexp) < 1e-15


def pin_finite_differences(impl):
    """Central differences of f = sum(O * dO), h = 1e-6, N <= 16, d <= 8,
    causal and not, g in {1, 2}: agreement to 1e-6 relative."""
    h = 1e-6
    for causal in (False, True):
        for (hq, hkv) in ((1, 1), (2, 1)):
            n, d = 6, 3
            q, k, v, do = rnd(1, hq, n, d), rnd(1, hkv, n, d), rnd(1, hkv, n, d), rnd(1, hq, n, d)
            sc = 0.8
            dq, dk, dv, _ = impl.backward(q, k, v, do, sc, causal)

            def f(q_, k_, v_):
                return float(np.sum(impl.forward(q_, k_, v_, sc, causal)[0] * do))

            for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
                num = np.zeros_like(x)
                it = np.nditer(x, flags=["multi_index"])
                for _ in it:
                    idx = it.multi_index
                    xp, xm = x.copy(), x.copy()
                    xp[idx] += h
                    xm[idx] -= h
                    args_p = {"q": q, "k": k, "v": v}
                    args_m = dict(args_p)
                    args_p[name], args_m[name] = xp, xm
                    num[idx] = (f(args_p["q"], args_p["k"], args_p["v"]) -
                                f(args_m["q"], args_m["k"], args_m["v"])) / (2 * h)
                err = np.linalg.norm(num - g) / max(np.linalg.norm(num), 1e-300)
                assert err < 1e-6, (name, causal, hq, err)


def pin_torch_sdpa(impl):
    """Second opinion: torch's float64 CPU scaled_dot_product_attention and its
    autograd (the routine the blog section 5 and the CSDN test compare to)."""
    import torch.nn.functional as F
    for causal in (False, True):
        for (hq, hkv) in ((2, 2), (4, 2)):
            q, k, v, do = rnd(2, hq, 17, 8), rnd(2, hkv, 17, 8), rnd(2, hkv, 17, 8), rnd(2, hq, 17, 8)
            tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
            to = F.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=0.35,
                                                enable_gqa=(hq != hkv))
            to.backward(torch.tensor(do))
            o, lse = impl.forward(q, k, v, 0.35, causal)
            dq, dk, dv, _ = impl.backward(q, k, v, do, 0.35, causal)
            np.testing.assert_allclose(o, to.detach().numpy(), atol=1e-12)
            np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-11)
            np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-11)
            np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-11)
            kk = torch.tensor(k).repeat_interleave(hq // hkv, dim=1)
            s = 0.35 * torch.tensor(q) @ kk.transpose(-1, -2)
            if causal:
                s = s.masked_fill(torch.ones(17, 17, dtype=torch.bool).triu(1), float("-inf"))
            np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), atol=1e-12)


def pin_row_forms(impl):
    """The row-subset forms equal the full forms on the chosen rows."""
    for causal in (False, True):
        q, k, v, do = rnd(1, 4, 40, 5), rnd(1, 2, 40, 5), rnd(1, 2, 40, 5), rnd(1, 4, 40, 5)
        o, lse = impl.forward(q, k, v, 0.45, causal)
        dq, dk, dv, D = impl.backward(q, k, v, do, 0.45, causal)
        rows = np.array([0, 3, 17, 39])
        for h in range(4):
            kh = h // 2
            orow, lrow = impl.forward_rows(q[0, h], k[0, kh], v[0, kh], 0.45, causal, rows)
            np.testing.assert_allclose(orow, o[0, h, rows], atol=1e-13)
            np.testing.assert_allclose(lrow, lse[0, h, rows], atol=1e-13)
            np.testing.assert_allclose(impl.lse_rows(q[0, h], k[0, kh], 0.45, causal, rows, chunk=3),
                                       lse[0, h, rows], atol=1e-13)
            dqr, Dr = impl.backward_rows(q[0, h], k[0, kh], v[0, kh], do[0, h], 0.45, causal, rows)
            np.testing.assert_allclose(dqr, dq[0, h, rows], atol=1e-12)
            np.testing.assert_allclose(Dr, D[0, h, rows], atol=1e-12)
        kv_rows = np.array([1, 20, 38])
        for kh in range(2):
            dkr, dvr = impl.backward_kv_rows([q[0, 2 * kh], q[0, 2 * kh + 1]], k[0, kh], v[0, kh],
                                             [do[0, 2 * kh], do[0, 2 * kh + 1]], 0.45, causal,
                                             kv_rows, chunk=7)
            np.testing.assert_allclose(dkr, dk[0, kh, kv_rows], atol=1e-12)
            np.testing.assert_allclose(dvr, dv[0, kh, kv_rows], atol=1e-12)


def pin_bottom_right(impl):
    """Bottom-right causal alignment (key j hidden from query i when
    j > i + Nk - Nq): a single query sees every key (= non-causal); the Nq
    queries equal the last Nq rows of the square top-left problem whatever
    precedes them; offset 0 is the top-left mask."""
    nk, d = 11, 4
    k, v = rnd(1, 1, nk, d), rnd(1, 1, nk, d)
    q1 = rnd(1, 1, 1, d)
    o_c, l_c = impl.forward(q1, k, v, 0.6, True, nk - 1)
    o_n, l_n = impl.forward(q1, k, v, 0.6, False)
    np.testing.assert_allclose(o_c, o_n, atol=1e-14)
    np.testing.assert_allclose(l_c, l_n, atol=1e-14)
    for nq in (3, 7, nk):
        q = rnd(1, 1, nq, d)
        qpad = np.concatenate([rnd(1, 1, nk - nq, d), q], axis=2)
        o_sq, l_sq = impl.forward(qpad, k, v, 0.6, True)
        o_br, l_br = impl.forward(q, k, v, 0.6, True, nk - nq)
        np.testing.assert_allclose(o_br, o_sq[:, :, nk - nq:], atol=1e-13)
        np.testing.assert_allclose(l_br, l_sq[:, :, nk - nq:], atol=1e-13)
        p = impl.probs(q[0, 0], k[0, 0], 0.6, True, nk - nq)
        i, j = np.meshgrid(np.arange(nq), np.arange(nk), indexing="ij")
        assert np.all(p[j > i + nk - nq] == 0) and np.all(p[j <= i + nk - nq] > 0)


def pin_merge_partials(impl):
    """Split-KV: pieces over any cut of the key range (empty pieces, one-key
    pieces, pieces a causal row cannot see) merge to the one-shot result; the
    two-piece merge equals its closed form; piece order does not matter."""
    nq, nk, d = 6, 19, 4
    q, k, v = rnd(2, 2, nq, d), rnd(2, 1, nk, d), rnd(2, 1, nk, d)
    for causal, off in ((False, 0), (True, nk - nq)):
        o, l = impl.forward(q, k, v, 0.5, causal, off)
        for bounds in ([0, nk], [0, 1, nk], [0, 5, 5, 12, 18, nk], [0, 15, 17, nk]):
            o_s, l_s, op, lp = impl.splitkv_forward(q, k, v, 0.5, causal, bounds, off)
            np.testing.assert_allclose(o_s, o, atol=1e-13)
            np.testing.assert_allclose(l_s, l, atol=1e-13)
            perm = np.arange(len(bounds) - 1)[::-1]
            o_p, l_p = impl.merge_partials(op[perm], lp[perm])
            np.testing.assert_allclose(o_p, o, atol=1e-13)
            np.testing.assert_allclose(l_p, l, atol=1e-13)
    o1, o2 = rnd(3, d), rnd(3, d)
    l1, l2 = rnd(3), rnd(3)
    om, lm = impl.merge_partials(np.stack([o1, o2]), np.stack([l1, l2]))
    w1, w2 = np.exp(l1), np.exp(l2)
    np.testing.assert_allclose(om, (w1[:, None] * o1 + w2[:, None] * o2) / (w1 + w2)[:, None],
                               atol=1e-14)
    np.testing.assert_allclose(lm, np.log(w1 + w2), atol=1e-14)
    oe, le = impl.merge_partials(np.stack([o1, np.zeros_like(o1)]),
                                 np.stack([l1, np.full(3, -np.inf)]))
    np.testing.assert_allclose(oe, o1, atol=1e-15)
    np.testing.assert_allclose(le, l1, atol=1e-15)


PINS = [pin_probs_rows, pin_constant_v, pin_causal_row0, pin_zero_q, pin_single_key,
        pin_shift_invariance, pin_kplus8_bf16, pin_gradient_identities, pin_permutation,
        pin_hand_example, pin_finite_differences, pin_torch_sdpa, pin_row_forms,
        pin_bottom_right, pin_merge_partials]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin(real_impl())


# ---------------------------------------------------------------------------
# the block-wise recurrences (blog section 2.2 and 4.1) equal the one-shot softmax
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("block", [1, 3, 7, 256, 300])
def test_blockwise_equals_one_shot(block, causal):
    n = 300
    q, k, v = rnd(n, 8), rnd(n, 8), rnd(n, 8)
    o, lse = OA.forward(q[None, None], k[None, None], v[None, None], 8 ** -0.5, causal)
    for fn in (OA.blockwise_forward_v1, OA.blockwise_forward_v2):
        ob, lb = fn(q, k, v, 8 ** -0.5, causal, block)
        np.testing.assert_allclose(ob, o[0, 0], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lb, lse[0, 0], rtol=1e-12, atol=1e-12)


def test_csdn_worked_setup():
    """The CSDN tutorial's own test: batch 2, length 1024, d 64, block 256; the
    block-wise result equals standard attention up to float rounding."""
    cfg = json.load(open(os.path.join(GOLDEN, "csdn_blockwise_test.json")))
    import attn_inputs
    t = attn_inputs.draw(cfg["batch"], 1, 1, cfg["seq_len"], cfg["seq_len"], cfg["d_k"], seed=2,
                         dtype=torch.float32)
    q, k, v = (attn_inputs.as_f64(t[n]) for n in ("q", "k", "v"))
    o, lse = OA.forward(q, k, v, cfg["scale"], cfg["causal"])
    for b in range(cfg["batch"]):
        ob, lb = OA.blockwise_forward_v2(q[b, 0], k[b, 0], v[b, 0], cfg["scale"], cfg["causal"],
                                         cfg["block_size"])
        assert np.max(np.abs(ob - o[b, 0])) < 1e-12
        assert np.max(np.abs(lb - lse[b, 0])) < 1e-12


def test_blog_s_size():
    """The blog's IO example: the N x N score matrix of one head at N = 4096 in
    FP16 is 4096*4096*2 bytes (~32 MB); the oracle materialises exactly that
    shape."""
    cfg = json.load(open(os.path.join(GOLDEN, "blog_s_matrix_size.json")))
    n = cfg["N"]
    s = OA.scores(np.zeros((n, 1)), np.zeros((n, 1)), 1.0, False)
    assert s.shape == (n, n)
    assert s.size * cfg["bytes_per_element"] == cfg["s_bytes"]


# ---------------------------------------------------------------------------
# planted mistakes: each must fail at least one pin
# ---------------------------------------------------------------------------

def _mutant(name):
    impl = real_impl()
    patches = {}
    if name == "mask_includes_diagonal":
        patches["_causal_mask"] = lambda nq, nk, offset=0: (np.arange(nk)[None, :] >=
                                                            np.arange(nq)[:, None] + offset)
    elif name == "mask_off_by_one_late":
        patches["_causal_mask"] = lambda nq, nk, offset=0: (np.arange(nk)[None, :] >
                                                            np.arange(nq)[:, None] + offset + 1)
    elif name == "scale_dropped":
        orig = OA.scores
        patches["scores"] = lambda q2, k2, scale, causal, off=0: orig(q2, k2, 1.0, causal, off)
    elif name == "lse_log2":
        f = impl.forward

        def fwd(*a):
            o, l = f(*a)
            return o, l / math.log(2)
        impl.forward = fwd
    elif name == "dk_no_scale":
        b = impl.backward

        def bwd(q, k, v, do, scale, causal):
            dq, dk, dv, D = b(q, k, v, do, scale, causal)
            return dq, dk / scale, dv, D
        impl.backward = bwd
    elif name == "dv_untransposed":
        b = impl.backward

        def bwd(q, k, v, do, scale, causal):
            dq, dk, dv, D = b(q, k, v, do, scale, causal)
            return dq, dk, dv[:, :, ::-1].copy(), D
        impl.backward = bwd
    elif name == "causal_offset_ignored":
        patches["_causal_mask"] = lambda nq, nk, offset=0: (np.arange(nk)[None, :] >
                                                            np.arange(nq)[:, None])
    elif name == "merge_unweighted":
        def merge(o_parts, lse_parts):
            o_parts, lse_parts = np.asarray(o_parts), np.asarray(lse_parts)
            m = np.max(lse_parts, axis=0)
            return o_parts.mean(axis=0), m + np.log(np.sum(np.exp(lse_parts - m), axis=0))
        patches["merge_partials"] = merge
        impl.merge_partials = merge
    elif name == "gqa_mod_mapping":
        patches["_kv_head"] = lambda h, hq, hkv: h % hkv
    elif name == "D_without_O":
        b = impl.backward

        def bwd(q, k, v, do, scale, causal):
            q_, k_, v_, do_ = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
            dq, dk, dv, D = b(q_, k_, v_, do_, scale, causal)
            # plant: dS computed with D = rowsum(dO) instead of rowsum(dO*O)
            D2 = do_.sum(axis=-1)
            B, Hq, Nq, d = q_.shape
            Hkv = k_.shape[1]
            dq2 = np.zeros_like(q_)
            dk2 = np.zeros_like(k_)
            for bb in range(B):
                for h in range(Hq):
                    kh = h // (Hq // Hkv)
                    p = OA.probs(q_[bb, h], k_[bb, kh], scale, causal)
                    dp = do_[bb, h] @ v_[bb, kh].T
                    ds = p * (dp - D2[bb, h][:, None])
                    dq2[bb, h] = scale * ds @ k_[bb, kh]
                    dk2[bb, kh] += scale * ds.T @ q_[bb, h]
            return dq2, dk2, dv, D2
        impl.backward = bwd
    elif name == "no_max_subtraction_overflow":
        # softmax without the max shift overflows for large scores -> NaN
        def pr(q2, k2, scale, causal, off=0):
            s = OA.scores(q2, k2, scale, causal, off) * 1e3
            e = np.exp(s)
            return e / e.sum(axis=1, keepdims=True)
        impl.probs = pr
    else:
        raise KeyError(name)
    return impl, patches


MUTANTS = ["mask_includes_diagonal", "mask_off_by_one_late", "scale_dropped", "lse_log2",
           "dk_no_scale", "dv_untransposed", "gqa_mod_mapping", "D_without_O",
           "no_max_subtraction_overflow", "causal_offset_ignored", "merge_unweighted"]


@pytest.mark.parametrize("mutant", MUTANTS)
def test_pins_catch_mutants(mutant, monkeypatch):
    impl, patches = _mutant(mutant)
    for k, v in patches.items():
        monkeypatch.setattr(OA, k, v)
    caught = []
    with np.errstate(all="ignore"):
        for pin in PINS:
            try:
                pin(impl)
            except (AssertionError, ValueError, FloatingPointError):
                caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {mutant}"
