"""GPU parity of the causal forward on the shapes where its unit order
changes: bf16 d = 256 with more than 256 MB of K and V, where the heads go in
groups (heaviest query blocks first inside each group, the last group
smaller).  Rows of every head, several query blocks each, are compared with
the float64 oracle, so a unit that the grouped order left out or took twice
would show."""
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


@pytest.mark.parametrize("shape", [
    # B, Hq, Hkv, N: K/V 268 MB at d = 256
    (1, 67, 67, 4096),    # groups of 12 heads, the last one of 7
    (1, 134, 67, 2048),   # GQA: groups of 24 query heads (12 key/value heads), last of 14
], ids=lambda s: "x".join(map(str, s)))
def test_grouped_causal_order_every_head(shape):
    B, Hq, Hkv, N = shape
    d = 256
    x = attn_inputs.draw(B, Hq, Hkv, N, N, d, 41, torch.bfloat16)
    g = to_dev(x)
    scale = d ** -0.5
    o, lse = F.forward(g["q"], g["k"], g["v"], scale, True)
    torch.cuda.synchronize()
    assert F.fa_device_status() == F.FA_OK
    assert bool(torch.isfinite(o).all()) and bool(torch.isfinite(lse).all())
    rng = np.random.default_rng(42)
    gq = Hq // Hkv
    for h in range(Hq):
        # one row in each of four query-block quarters of the sequence
        rows = np.array(sorted({int(rng.integers(k * N // 4, (k + 1) * N // 4)) for k in range(4)}))
        o_ref, l_ref = oracle.forward_rows(f64(x["q"][0, h]), f64(x["k"][0, h // gq]),
                                           f64(x["v"][0, h // gq]), scale, True, rows)
        check_o(f64(o[0, h][rows]), o_ref, "bf16")
        check_l(f64(lse[0, h][rows]), l_ref, "bf16")
