"""GPU parity of the split-KV forward (fa_fwd_splitkv): pieces of the key
range computed by separate CTAs and merged by their log-sum-exp, with the
causal mask bottom-right aligned when Nq < Nk.  Compared element by element
with the float64 oracle (forward with causal_offset = Nk - Nq) on seeded
inputs, and on sampled rows at the inference workload's full size."""
import numpy as np
import pytest
import torch

import attn_inputs
import exact_io_aware_50_b200 as F
import oracle
from parity import check_l, check_o, f64, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    F.lib()
    yield


# (B, Hq, Hkv, Nq, Nk, d, causal, num_splits); num_splits None = library's choice
CASES = [
    (1, 2, 1, 1, 1000, 128, True, 3),       # one query row: sees every key
    (1, 4, 2, 200, 1111, 64, True, 5),      # GQA, ragged tails on both axes
    (2, 2, 2, 129, 700, 128, False, 4),
    (1, 2, 2, 300, 300, 256, True, 2),      # Nq == Nk: the top-left mask of fa_fwd
    (1, 1, 1, 64, 4096, 128, True, 64),     # more pieces than visible key blocks
    (1, 3, 1, 257, 2000, 128, True, 1),     # one piece: plain kernel, shifted mask
    (1, 2, 2, 96, 5000, 64, False, None),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(str(v) for v in c))
def test_splitkv_small(case):
    B, Hq, Hkv, Nq, Nk, d, causal, splits = case
    x = attn_inputs.draw(B, Hq, Hkv, Nq, Nk, d, seed=900 + Nq + Nk)
    g = to_dev(x)
    o, lse = F.forward_splitkv(g["q"], g["k"], g["v"], d ** -0.5, causal, splits)
    torch.cuda.synchronize()
    assert F.fa_device_status() == F.FA_OK
    o_ref, l_ref = oracle.forward(f64(x["q"]), f64(x["k"]), f64(x["v"]), d ** -0.5, causal,
                                  Nk - Nq if causal else 0)
    check_o(f64(o), o_ref, "bf16")
    check_l(f64(lse), l_ref, "bf16")


def test_splitkv_matches_fa_fwd_when_square():
    """Nq == Nk, causal: the split path equals the oracle (top-left and
    bottom-right causal coincide here) and agrees with fa_fwd to the
    rounding of a different summation order."""
    x = attn_inputs.draw(1, 4, 4, 1024, 1024, 128, seed=77)
    g = to_dev(x)
    o1, l1 = F.forward(g["q"], g["k"], g["v"], 128 ** -0.5, True)
    o2, l2 = F.forward_splitkv(g["q"], g["k"], g["v"], 128 ** -0.5, True, 4)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.forward(*(f64(x[n]) for n in ("q", "k", "v")), 128 ** -0.5, True)
    check_o(f64(o2), o_ref, "bf16")
    check_l(f64(l2), l_ref, "bf16")
    # different rounding order: allow one bf16 ulp of O
    assert float(((o1.float() - o2.float()).abs() / o1.float().abs().clamp(min=1.0)).max()) <= 2.0 ** -7
    assert float((l1 - l2).abs().max()) <= 1e-4


def test_inference_workload_sampled():
    w = attn_inputs.INFER_PREFILL
    x = attn_inputs.make(w)
    g = to_dev(x)
    n_split = F.fa_fwd_splitkv_num_splits(w.B, w.Hq, w.Nq, w.Nk, w.d)
    assert n_split > 1
    o, lse = F.forward_splitkv(g["q"], g["k"], g["v"], w.scale, w.causal, n_split)
    torch.cuda.synchronize()
    assert F.fa_device_status() == F.FA_OK
    assert bool(torch.isfinite(o).all()) and bool(torch.isfinite(lse).all())
    rng = np.random.default_rng(w.seed)
    rows = np.array(sorted(set(rng.choice(w.Nq, 24, replace=False).tolist()) | {0, 255, 256, w.Nq - 1}))
    for h in (0, w.Hq - 1):
        q2, k2, v2 = f64(x["q"][0, h]), f64(x["k"][0, h]), f64(x["v"][0, h])
        o_ref, l_ref = oracle.forward_rows(q2, k2, v2, w.scale, True, rows, causal_offset=w.Nk - w.Nq)
        check_o(f64(o[0, h][rows]), o_ref, "bf16")
        check_l(f64(lse[0, h][rows]), l_ref, "bf16")
