"""GPU parity of dropout on P (fa_fwd_dropout / fa_bwd_dropout) against the
float64 oracle with the same Philox4x32-10 mask: the mask itself read back
bit for bit, forward and backward element by element on small seeded cases,
p = 0 equal to the plain path bit for bit, and sampled rows at the training
workload's full size."""
import numpy as np
import pytest
import torch

import attn_inputs
import exact_io_aware_50_b200 as F
import oracle
from parity import check_grad, check_l, check_o, f64, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    F.lib()
    yield


def test_dropout_mask_bits():
    """Q = 0 makes P uniform; V = identity rows makes O_ij = Z_ij / (Nk (1 - p)),
    so the kernel's keep mask can be read off O and compared with the oracle's
    bit for bit (all heads, causal and not)."""
    B, Hq, Nk, d, p, seed, off = 2, 3, 64, 128, 0.3, 0x1234_5678_9abc, 5
    for causal in (False, True):
        q = torch.zeros(B, Hq, Nk, d, dtype=torch.bfloat16)
        v = torch.zeros(B, Hq, Nk, d, dtype=torch.bfloat16)
        for j in range(Nk):
            v[:, :, j, j] = 1.0
        k = attn_inputs.draw(B, Hq, Hq, Nk, Nk, d, seed=3)["k"]
        o, _ = F.forward_dropout(q.cuda(), k.cuda(), v.cuda(), p, seed, off, causal=causal)
        torch.cuda.synchronize()
        o = f64(o)
        for b in range(B):
            for h in range(Hq):
                z = oracle.dropout_keep(b * Hq + h, np.arange(Nk), np.arange(Nk), p, seed, off)
                if causal:
                    z = z & (np.arange(Nk)[None, :] <= np.arange(Nk)[:, None])
                got = o[b, h][:, :Nk] > 0
                assert np.array_equal(got, z), f"mask differs at b={b} h={h} causal={causal}"


CASES = [(1, 2, 1, 300, 64, True, 0.1), (2, 2, 2, 257, 128, False, 0.5),
         (1, 4, 2, 513, 128, True, 0.3), (1, 2, 1, 300, 256, True, 0.2),
         (2, 2, 2, 200, 256, False, 0.4),
         # more units than SMs: the mask warps and the readout warps' mask
         # cursors cross unit boundaries, and the d = 256 passes run persistently
         (24, 4, 2, 400, 128, True, 0.2), (24, 4, 2, 400, 64, True, 0.1),
         (32, 4, 2, 400, 256, False, 0.3)]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(str(v) for v in c))
def test_dropout_small(case):
    B, Hq, Hkv, N, d, causal, p = case
    seed, off = 987654321, 3
    x = attn_inputs.draw(B, Hq, Hkv, N, N, d, seed=42 + N)
    g = to_dev(x)
    o, lse = F.forward_dropout(g["q"], g["k"], g["v"], p, seed, off, causal=causal)
    dq, dk, dv = F.backward_dropout(g["q"], g["k"], g["v"], o, lse, g["do"], p, seed, off,
                                    causal=causal)
    torch.cuda.synchronize()
    assert F.fa_device_status() == F.FA_OK
    qf, kf, vf, dof = (f64(x[n]) for n in ("q", "k", "v", "do"))
    o_ref, l_ref = oracle.dropout_forward(qf, kf, vf, d ** -0.5, causal, p, seed, off)
    check_o(f64(o), o_ref, "bf16")
    check_l(f64(lse), l_ref, "bf16")
    # the backward is checked against the oracle's gradients at the kernel's own O
    dq_r, dk_r, dv_r, _ = oracle.dropout_backward(qf, kf, vf, dof, d ** -0.5, causal, p, seed, off)
    check_grad(f64(dq), dq_r, "bf16", "dQ")
    check_grad(f64(dk), dk_r, "bf16", "dK")
    check_grad(f64(dv), dv_r, "bf16", "dV")


def test_dropout_p0_is_plain():
    x = attn_inputs.draw(1, 2, 2, 384, 384, 128, seed=5)
    g = to_dev(x)
    o1, l1 = F.forward(g["q"], g["k"], g["v"], None, True)
    o2, l2 = F.forward_dropout(g["q"], g["k"], g["v"], 0.0, 77, 0, causal=True)
    g1 = F.backward(g["q"], g["k"], g["v"], o1, l1, g["do"], None, True)
    g2 = F.backward_dropout(g["q"], g["k"], g["v"], o1, l1, g["do"], 0.0, 77, 0, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


def test_dropout_training_workload_sampled():
    w = attn_inputs.CAUSAL_TRAIN
    p, seed, off = 0.1, 2026, 11
    x = attn_inputs.make(w)
    g = to_dev(x)
    o, lse = F.forward_dropout(g["q"], g["k"], g["v"], p, seed, off, w.scale, w.causal)
    dq, dk, dv = F.backward_dropout(g["q"], g["k"], g["v"], o, lse, g["do"], p, seed, off,
                                    w.scale, w.causal)
    torch.cuda.synchronize()
    assert F.fa_device_status() == F.FA_OK
    for t in (o, lse, dq, dk, dv):
        assert bool(torch.isfinite(t).all())
    rng = np.random.default_rng(w.seed)
    for b, h in ((0, 0), (w.B - 1, w.Hq - 1)):
        bh = b * w.Hq + h
        rows = np.array(sorted(set(rng.choice(w.N, 12, replace=False).tolist()) | {0, w.N - 1}))
        q2, k2, v2, do2 = (f64(x[n][b, h]) for n in ("q", "k", "v", "do"))
        o_ref, l_ref = oracle.dropout_forward_rows(q2, k2, v2, w.scale, True, rows, bh, p, seed, off)
        check_o(f64(o[b, h][rows]), o_ref, "bf16")
        check_l(f64(lse[b, h][rows]), l_ref, "bf16")
        dq_ref, _ = oracle.dropout_backward_rows(q2, k2, v2, do2, w.scale, True, rows, bh, p, seed,
                                                 off)
        # Causal row 0 sees one key: its exact dQ is 0 (dS_00 = P_00 (dP_00 - D_0) = 0).
        # The backward takes D = rowsum(dO * O) from the caller's bf16 O, and with
        # dropout O_0 = Z V_0 / (1 - p) is not a bf16 number, so |dQ_0| is bounded
        # by the output rounding instead: scale * |dD| * |K_0 - c|, with
        # |dD| <= sum_d |dO_0d| ulp(O_0d) / 2 and |c_d| <= |mean of K's first 64
        # rows|_d + 1/2 (c is that mean rounded to integers).
        assert rows[0] == 0 and np.all(dq_ref[0] == 0.0)
        half_ulp = np.ldexp(1.0, np.floor(np.log2(np.maximum(np.abs(o_ref[0]), 2.0 ** -126))).astype(int) - 8)
        d_bound = np.sum(np.abs(do2[0]) * half_ulp)
        c_bound = np.abs(k2[:64].mean(axis=0)) + 0.5
        k_bound = np.linalg.norm(np.abs(k2[0]) + c_bound)
        assert np.linalg.norm(f64(dq[b, h][0])) <= w.scale * d_bound * k_bound
        check_grad(f64(dq[b, h][rows[1:]]), dq_ref[1:], "bf16", "dQ rows")
        kv_rows = np.array([0, 1000, w.N - 1])
        dk_ref, dv_ref = oracle.dropout_backward_kv_rows([q2], k2, v2, [do2], [bh], w.scale, True,
                                                         kv_rows, p, seed, off)
        check_grad(f64(dk[b, h][kv_rows]), dk_ref, "bf16", "dK rows")
        check_grad(f64(dv[b, h][kv_rows]), dv_ref, "bf16", "dV rows")
