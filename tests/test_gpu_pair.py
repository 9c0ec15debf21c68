"""GPU parity of the CTA-pair forward (fa_fwd_pair: two CTAs share each
tile's tcgen05 MMAs, M = 256, each loading half of every K and V tile)
against the float64 oracle: whole tensors on shapes that span several pair
units, ragged tails (a pair's second CTA past the last query row, a key
block's second half past the last key), GQA groups, more units than pairs
(the persistent loop), and sampled rows at a full-size shape; plus the
argument checks of the entry point."""
import numpy as np
import pytest
import torch

import attn_inputs
import exact_io_aware_50_b200 as F
import oracle
from parity import check_l, check_o, f64, run_full_check, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    F.lib()
    yield


PAIR_SHAPES = [
    # B, Hq, Hkv, Nq, Nk, d, causal
    (1, 1, 1, 128, 128, 128, False),     # one pair, second CTA's rows all past the end
    (1, 1, 1, 512, 512, 128, True),
    (1, 1, 1, 1, 1, 128, False),
    (1, 2, 1, 300, 300, 128, True),      # ragged: 300 = 256 + 44
    (1, 2, 2, 17, 200, 128, False),      # key tail inside the second half of a block
    (2, 4, 2, 1000, 1000, 128, True),
    (1, 2, 1, 640, 384, 128, False),
    (1, 1, 1, 200, 1000, 256, False),
    (2, 2, 1, 513, 513, 256, True),
    (1, 4, 4, 256, 70, 256, False),      # keys end inside the first half of the block
    (16, 8, 4, 600, 600, 128, True),     # 384 units: several rounds per pair
    (8, 8, 8, 700, 700, 256, False),     # 192 units at d = 256
]


@pytest.mark.parametrize("shape", PAIR_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_pair_forward_matches_oracle(shape):
    B, Hq, Hkv, Nq, Nk, d, causal = shape
    run_full_check(B, Hq, Hkv, Nq, Nk, d, causal, "bf16", seed=31, backward=False, cta_pair=True)


@pytest.mark.parametrize("d", [128, 256])
def test_pair_forward_sharp_and_shifted(d):
    # Q x 2 sharpens the softmax; K + 8 moves every score of a row by the
    # same amount and stresses the running-max rescale (the cases the
    # single-CTA forward is held to)
    run_full_check(1, 4, 1, 1024, 1024, d, True, "bf16", seed=31, q_mul=2.0, backward=False,
                   cta_pair=True)
    run_full_check(1, 2, 2, 700, 700, d, False, "bf16", seed=32, k_add=8.0, backward=False,
                   cta_pair=True)


def test_pair_forward_equals_single_cta_closely():
    # both forms compute the same sums in the same per-row order of key
    # blocks; only the MMA split differs, so they agree to bf16 rounding
    x = attn_inputs.draw(2, 4, 2, 777, 777, 128, 33, torch.bfloat16, 1.0, 0.0)
    g = to_dev(x)
    o1, l1 = F.forward(g["q"], g["k"], g["v"], None, True)
    o2, l2 = F.forward(g["q"], g["k"], g["v"], None, True, cta_pair=True)
    torch.cuda.synchronize()
    assert F.fa_device_status() == F.FA_OK
    assert float((o1.float() - o2.float()).abs().max()) <= 2 ** -8
    assert float((l1 - l2).abs().max()) <= 1e-5


@pytest.mark.parametrize("d,causal", [(128, True), (256, False)])
def test_pair_forward_full_size_sampled(d, causal):
    # B4 H16 N4096: 512 / 1024 units over the GPU's pairs
    B, H, N = 4, 16, 4096
    x = attn_inputs.draw(B, H, H, N, N, d, 34, torch.bfloat16, 1.0, 0.0)
    g = to_dev(x)
    scale = d ** -0.5
    o, lse = F.forward(g["q"], g["k"], g["v"], scale, causal, cta_pair=True)
    torch.cuda.synchronize()
    assert F.fa_device_status() == F.FA_OK
    assert bool(torch.isfinite(o).all()) and bool(torch.isfinite(lse).all())
    rng = np.random.default_rng(35)
    for b, h in [(0, 0), (B - 1, H - 1), (int(rng.integers(B)), int(rng.integers(H)))]:
        rows = np.unique(np.concatenate([rng.integers(0, N, 20), [0, 127, 128, 255, 256, N - 1]]))
        o_ref, l_ref = oracle.forward_rows(f64(x["q"][b, h]), f64(x["k"][b, h]), f64(x["v"][b, h]),
                                           scale, causal, rows)
        check_o(f64(o[b, h][rows]), o_ref, "bf16")
        check_l(f64(lse[b, h][rows]), l_ref, "bf16")


def test_pair_forward_rejects_d64_and_float32():
    q = torch.zeros(1, 1, 128, 64, device="cuda", dtype=torch.bfloat16)
    o = torch.empty_like(q)
    lse = torch.empty(1, 1, 128, device="cuda", dtype=torch.float32)
    st = F.fa_fwd_pair(q.data_ptr(), q.data_ptr(), q.data_ptr(), o.data_ptr(), lse.data_ptr(),
                       1, 1, 1, 128, 128, 64, 0.125, 0)
    assert st == F.FA_ERR_UNSUPPORTED
    with pytest.raises(ValueError):
        F.forward(q.float(), q.float(), q.float(), cta_pair=True)
