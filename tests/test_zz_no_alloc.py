"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory
where they call it (the scratch lives in a fixed array inside the library).

The GPU test calls the entry point through the C ABI twice in a row and
compares each result with fa_bwd (the workspace entry point) on the same
inputs, within the gradient tolerance of the parity tests.  This file is named
to be collected last, so a run that stops at the first failure has already
run every other test.
"""
import ctypes

import pytest
import torch

import attn_inputs
import exact_io_aware_50_b200 as F
from parity import GRAD_REL_TOL

FAKE = 1 << 20  # aligned, non-null, never dereferenced (the call is refused first)


def _noalloc():
    fn = F.lib().fa_bwd_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [P] * 9 + [I, I, I, I, I, I, ctypes.c_float, I, P]
    fn.restype = I
    return fn


def test_noalloc_refuses_problems_larger_than_its_scratch():
    # 4 * 1 * 32 * 16384 * 129 bytes > 32 MiB: refused before any device work
    st = _noalloc()(*([FAKE] * 9), 1, 32, 8, 16384, 16384, 128, 0.088, 1, None)
    assert st == F.FA_ERR_UNSUPPORTED
    assert _noalloc()(*([0] + [FAKE] * 8), 1, 1, 1, 8, 8, 64, 0.125, 0, None) == F.FA_ERR_INVALID_ARG


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [(1, 4, 2, 1000, 128, True), (2, 2, 2, 700, 64, False),
                                   (1, 2, 2, 512, 256, True)])
def test_noalloc_matches_workspace_backward_twice(shape):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B, Hq, Hkv, N, d, causal = shape
    x = attn_inputs.draw(B, Hq, Hkv, N, N, d, seed=91)
    g = {k: v.cuda() for k, v in x.items()}
    scale = d ** -0.5
    o, lse = F.forward(g["q"], g["k"], g["v"], scale, causal)
    dq_ref, dk_ref, dv_ref = F.backward(g["q"], g["k"], g["v"], o, lse, g["do"], scale, causal)
    stream = torch.cuda.current_stream().cuda_stream
    fn = _noalloc()
    for _ in range(2):
        dq, dk, dv = torch.empty_like(g["q"]), torch.empty_like(g["k"]), torch.empty_like(g["v"])
        st = fn(g["q"].data_ptr(), g["k"].data_ptr(), g["v"].data_ptr(), o.data_ptr(),
                lse.data_ptr(), g["do"].data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                B, Hq, Hkv, N, N, d, scale, int(causal), stream)
        assert st == F.FA_OK, F.fa_strerror(st)
        torch.cuda.synchronize()
        assert F.fa_device_status() == F.FA_OK
        for got, ref, name in ((dq, dq_ref, "dQ"), (dk, dk_ref, "dK"), (dv, dv_ref, "dV")):
            rel = float((got.double() - ref.double()).norm() / ref.double().norm())
            assert rel <= GRAD_REL_TOL, f"{name}: relative error {rel:.3g} vs fa_bwd"
