"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/fa.h declares, and rejects bad arguments before
touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

import exact_io_aware_50_b200 as F

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_fwd_f32", "fa_bwd_f32",
              "fa_strerror", "fa_device_status", "fa_wait_selftest"):
        assert n in names


def test_library_exports_every_declared_symbol():
    L = F.lib()
    for n in declared_functions():
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", F.lib_path], capture_output=True,
                         text=True).stdout
    exported = set(re.findall(r" T (fa_\w+)", out))
    assert set(declared_functions()) <= exported
    # nothing but the ABI is exported as a function
    assert exported == set(declared_functions())


def test_strerror_covers_codes():
    for code in range(0, 7):
        assert F.fa_strerror(code) not in ("", "unknown status")
    assert F.fa_strerror(99) == "unknown status"


def _ws_expected(B, H, N, d):
    # D and L2 rows padded to 128 per head, the centring vectors, a 16-byte
    # work counter, then the 256-byte aligned f32 dQ accumulator
    npad = (N + 127) // 128 * 128
    head = 2 * B * H * npad * 4 + B * H * d * 4 + 16
    return (head + 255) // 256 * 256 + B * H * N * d * 4


def test_workspace_size():
    for (B, H, N, d) in ((4, 16, 4096, 128), (1, 1, 3, 64), (2, 3, 1000, 256), (1, 32, 16384, 128)):
        assert F.fa_bwd_workspace_size(B, H, N, d) == _ws_expected(B, H, N, d)
    assert F.fa_bwd_workspace_size(0, 1, 1, 64) == 0


FAKE = 1 << 20  # 16-byte aligned non-null address; never dereferenced (rejected first)


@pytest.mark.parametrize("fn", ["fa_fwd", "fa_fwd_f32", "fa_fwd_pair"])
def test_forward_argument_errors(fn):
    f = getattr(F, fn)
    ok = dict(B=1, Hq=2, Hkv=1, Nq=8, Nk=8, d=128 if fn == "fa_fwd_pair" else 64, scale=0.125,
              causal=0)

    def call(ptrs=(FAKE,) * 5, **kw):
        a = dict(ok)
        a.update(kw)
        return f(*ptrs, a["B"], a["Hq"], a["Hkv"], a["Nq"], a["Nk"], a["d"], a["scale"], a["causal"])

    assert call(ptrs=(0, FAKE, FAKE, FAKE, FAKE)) == F.FA_ERR_INVALID_ARG
    assert call(B=0) == F.FA_ERR_INVALID_ARG
    assert call(Nk=-1) == F.FA_ERR_INVALID_ARG
    assert call(Hq=3, Hkv=2) == F.FA_ERR_INVALID_ARG
    assert call(scale=0.0) == F.FA_ERR_INVALID_ARG
    assert call(scale=float("nan")) == F.FA_ERR_INVALID_ARG
    assert call(scale=float("inf")) == F.FA_ERR_INVALID_ARG
    assert call(causal=1, Nq=8, Nk=9) == F.FA_ERR_UNSUPPORTED
    if fn == "fa_fwd":
        assert call(d=96) == F.FA_ERR_UNSUPPORTED
        assert call(d=32) == F.FA_ERR_UNSUPPORTED
    elif fn == "fa_fwd_pair":
        assert call(d=64) == F.FA_ERR_UNSUPPORTED   # pairs split d in two 128-byte halves
        assert call(d=96) == F.FA_ERR_UNSUPPORTED
    else:
        assert call(d=260) == F.FA_ERR_UNSUPPORTED
        assert call(d=6) == F.FA_ERR_UNSUPPORTED
    assert call(ptrs=(FAKE + 2, FAKE, FAKE, FAKE, FAKE)) == F.FA_ERR_ALIGNMENT


@pytest.mark.parametrize("fn", ["fa_bwd", "fa_bwd_f32"])
def test_backward_argument_errors(fn):
    f = getattr(F, fn)

    def call(ptrs=(FAKE,) * 10, d=64, Hq=2, Hkv=1):
        return f(*ptrs, 1, Hq, Hkv, 8, 8, d, 0.125, 0)

    assert call(ptrs=(FAKE,) * 9 + (0,)) == F.FA_ERR_INVALID_ARG
    assert call(Hq=4, Hkv=3) == F.FA_ERR_INVALID_ARG
    assert call(d=100 if fn == "fa_bwd" else 300) == F.FA_ERR_UNSUPPORTED
    assert call(ptrs=(FAKE,) * 9 + (FAKE + 16,)) == F.FA_ERR_ALIGNMENT  # workspace needs 256 B
    assert call(ptrs=(FAKE,) * 6 + (FAKE + 8,) + (FAKE,) * 3) == F.FA_ERR_ALIGNMENT


def test_selftest_rejects_bad_limit():
    assert F.fa_wait_selftest(0) == F.FA_ERR_INVALID_ARG
    assert F.fa_wait_selftest(2_000_000_000) == F.FA_ERR_INVALID_ARG


def test_splitkv_argument_errors():
    f = F.fa_fwd_splitkv

    def call(ptrs=(FAKE,) * 6, Nq=8, Nk=16, d=64, causal=1, splits=2):
        return f(*ptrs, 1, 2, 1, Nq, Nk, d, 0.125, causal, splits)

    assert call(splits=0) == F.FA_ERR_INVALID_ARG
    assert call(splits=2000) == F.FA_ERR_INVALID_ARG
    assert call(ptrs=(FAKE,) * 5 + (0,)) == F.FA_ERR_INVALID_ARG   # workspace needed
    assert call(ptrs=(0,) + (FAKE,) * 5) == F.FA_ERR_INVALID_ARG
    assert call(Nq=17, Nk=16) == F.FA_ERR_UNSUPPORTED              # causal needs Nq <= Nk
    assert call(d=96) == F.FA_ERR_UNSUPPORTED
    assert call(ptrs=(FAKE,) * 5 + (FAKE + 16,)) == F.FA_ERR_ALIGNMENT   # workspace 256 B
    assert call(ptrs=(FAKE + 4,) + (FAKE,) * 5) == F.FA_ERR_ALIGNMENT


def test_splitkv_sizes():
    def ws(B, H, N, d, s):
        head = (s * B * H * N * d * 4 + 255) // 256 * 256
        return head + s * B * H * N * 4
    for (B, H, N, d, s) in ((1, 8, 512, 128, 19), (2, 3, 1000, 64, 7), (1, 1, 1, 256, 2)):
        assert F.fa_fwd_splitkv_workspace_size(B, H, N, d, s) == ws(B, H, N, d, s)
    assert F.fa_fwd_splitkv_workspace_size(1, 8, 512, 128, 1) == 0
    assert F.fa_fwd_splitkv_workspace_size(1, 8, 512, 128, 0) == 0
    # 16 units of 256 query rows -> floor(148 / 16) = 9 pieces (one wave)
    assert F.fa_fwd_splitkv_num_splits(1, 8, 512, 16384, 128) == 9
    # enough units already: one piece
    assert F.fa_fwd_splitkv_num_splits(4, 16, 4096, 4096, 128) == 1
    # capped at half the number of 128-key blocks
    assert F.fa_fwd_splitkv_num_splits(1, 1, 1, 1024, 128) == 4
    assert F.fa_fwd_splitkv_num_splits(0, 1, 1, 1024, 128) == 0


def test_dropout_argument_errors():
    def fwd(p, d=64, ptrs=(FAKE,) * 5):
        return F.fa_fwd_dropout(*ptrs, 1, 2, 1, 8, 8, d, 0.125, 0, p, 1, 0)

    def bwd(p, d=64):
        return F.fa_bwd_dropout(*(FAKE,) * 10, 1, 2, 1, 8, 8, d, 0.125, 0, p, 1, 0)

    for bad in (-0.1, 1.0, 1.5, float("nan")):
        assert fwd(bad) == F.FA_ERR_INVALID_ARG
        assert bwd(bad) == F.FA_ERR_INVALID_ARG
    assert fwd(0.1, ptrs=(0,) + (FAKE,) * 4) == F.FA_ERR_INVALID_ARG
    assert fwd(0.1, d=96) == F.FA_ERR_UNSUPPORTED
    assert bwd(0.1, d=96) == F.FA_ERR_UNSUPPORTED       # dropout backward: d = 64, 128, 256
    assert fwd(0.1, ptrs=(FAKE + 2,) + (FAKE,) * 4) == F.FA_ERR_ALIGNMENT


def test_fp8_argument_errors():
    def fwd(dq=0.5, dk=0.5, dv=0.5, d=128, ptrs=(FAKE,) * 5, scale=0.125, causal=0, B=1):
        return F.fa_fwd_fp8(*ptrs, B, 2, 1, 8, d, scale, dq, dk, dv, causal)

    for bad in (0.0, -1.0, float("nan"), float("inf")):
        assert fwd(dq=bad) == F.FA_ERR_INVALID_ARG
        assert fwd(dk=bad) == F.FA_ERR_INVALID_ARG
        assert fwd(dv=bad) == F.FA_ERR_INVALID_ARG
    assert fwd(scale=0.0) == F.FA_ERR_INVALID_ARG
    assert fwd(B=0) == F.FA_ERR_INVALID_ARG
    for i in range(5):
        ptrs = [FAKE] * 5
        ptrs[i] = 0
        assert fwd(ptrs=tuple(ptrs)) == F.FA_ERR_INVALID_ARG
    for d in (64, 96, 192, 512):
        assert fwd(d=d) == F.FA_ERR_UNSUPPORTED       # e4m3 forward: d = 128, 256
    for i in range(5):
        ptrs = [FAKE] * 5
        ptrs[i] = FAKE + 8
        assert fwd(ptrs=tuple(ptrs)) == F.FA_ERR_ALIGNMENT


def test_size_limits():
    """Sizes past the kernels' index arithmetic are refused before any launch."""
    f = F.fa_fwd
    big_n = (1 << 28) + 1
    assert f(*(FAKE,) * 5, 1, 1, 1, big_n, 8, 64, 0.125, 0) == F.FA_ERR_UNSUPPORTED
    assert f(*(FAKE,) * 5, 1, 1, 1, 8, big_n, 64, 0.125, 0) == F.FA_ERR_UNSUPPORTED
    # B*Hq*Nq*d above 4e12 elements
    assert f(*(FAKE,) * 5, 4096, 1024, 1024, 8192, 8, 128, 0.125, 0) == F.FA_ERR_UNSUPPORTED


def test_wrappers_reject_bad_tensors_before_the_library():
    """The Python wrappers check shapes, dtypes, devices and the workspace size
    and raise ValueError; nothing reaches the C entry points (CPU tensors)."""
    import torch
    bf = torch.bfloat16
    q = torch.zeros(1, 2, 8, 64, dtype=bf)
    k = torch.zeros(1, 1, 8, 64, dtype=bf)
    with pytest.raises(ValueError, match="k, v both"):
        F.forward(q, k, torch.zeros(1, 1, 9, 64, dtype=bf))
    with pytest.raises(ValueError, match="disagree on B or d"):
        F.forward(q, torch.zeros(1, 1, 8, 32, dtype=bf), torch.zeros(1, 1, 8, 32, dtype=bf))
    with pytest.raises(ValueError, match="share one dtype"):
        F.forward(q, k, k.float())
    with pytest.raises(ValueError, match="share one dtype"):
        F.forward(q.half(), k.half(), k.half())
    with pytest.raises(ValueError, match="CUDA tensors"):
        F.forward(q, k, k)
    with pytest.raises(ValueError, match="share one dtype"):
        F.forward_fp8(q, k, k, 1.0, 1.0, 1.0)
    q8 = torch.zeros(1, 2, 8, 128, dtype=torch.uint8)
    with pytest.raises(ValueError, match="Nq must equal Nk"):
        F.forward_fp8(q8, torch.zeros(1, 1, 16, 128, dtype=torch.uint8),
                      torch.zeros(1, 1, 16, 128, dtype=torch.uint8), 1.0, 1.0, 1.0)
    with pytest.raises(ValueError, match="CUDA tensors"):
        F.forward_fp8(q8, q8[:, :1].contiguous(), q8[:, :1].contiguous(), 1.0, 1.0, 1.0)
    lse = torch.zeros(1, 2, 8)
    with pytest.raises(ValueError, match="o and dout must have q's shape"):
        F.backward(q, k, k, q[:, :1], lse, q)
    with pytest.raises(ValueError, match="o and dout must have q's dtype"):
        F.backward(q, k, k, q.float(), lse, q)
    with pytest.raises(ValueError, match="lse must be float32"):
        F.backward(q, k, k, q, lse.double(), q)
    with pytest.raises(ValueError, match="lse must be float32"):
        F.backward_dropout(q, k, k, q, lse[:, :, :4], q, 0.1, 1)
    with pytest.raises(ValueError, match="CUDA tensors"):
        F.backward(q, k, k, q, lse, q)


class _FakeCuda:
    """Stands in for a contiguous CUDA tensor on device `idx` without holding
    memory; reaching the library through it fails the test."""

    def __init__(self, shape, dtype, idx):
        import torch
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.device = torch.device("cuda", idx)
        self.is_cuda = True

    def dim(self):
        return len(self.shape)

    def is_contiguous(self):
        return True

    def numel(self):
        n = 1
        for s in self.shape:
            n *= s
        return n

    def element_size(self):
        import torch
        return torch.empty(0, dtype=self.dtype).element_size()

    def data_ptr(self):
        raise AssertionError("a tensor on the wrong device reached the library")


def test_wrappers_reject_tensors_on_another_device():
    """Every tensor a wrapper passes (inputs, caller outputs, workspaces) must be
    on q's device: the library launches on the current device, which the
    wrappers make q's, so a tensor on another GPU is refused with ValueError
    before anything is allocated or launched (stand-in tensors, no GPU)."""
    import torch
    bf = torch.bfloat16

    def t(shape, idx, dtype=bf):
        return _FakeCuda(shape, dtype, idx)

    q0, k0, v0 = t((1, 2, 8, 64), 0), t((1, 1, 8, 64), 0), t((1, 1, 8, 64), 0)
    lse0 = t((1, 2, 8), 0, torch.float32)
    with pytest.raises(ValueError, match="q's device"):
        F.forward(q0, t((1, 1, 8, 64), 1), v0)
    with pytest.raises(ValueError, match="q's device"):
        F.forward(q0, k0, t((1, 1, 8, 64), 1))
    with pytest.raises(ValueError, match="q's device"):
        F.forward(q0, k0, v0, out=t((1, 2, 8, 64), 1), lse=lse0)
    with pytest.raises(ValueError, match="q's device"):
        F.forward(q0, k0, v0, out=t((1, 2, 8, 64), 0), lse=t((1, 2, 8), 1, torch.float32))
    with pytest.raises(ValueError, match="q's device"):
        F.backward(q0, k0, v0, q0, lse0, t((1, 2, 8, 64), 1))
    with pytest.raises(ValueError, match="q's device"):
        F.backward(q0, k0, v0, t((1, 2, 8, 64), 1), lse0, q0)
    ws1 = t((F.fa_bwd_workspace_size(1, 2, 8, 64),), 1, torch.uint8)
    with pytest.raises(ValueError, match="workspace must be on q's device"):
        F.backward(q0, k0, v0, q0, lse0, q0, workspace=ws1)
    with pytest.raises(ValueError, match="workspace must be on q's device"):
        F.backward_dropout(q0, k0, v0, q0, lse0, q0, 0.1, 1, workspace=ws1)
    with pytest.raises(ValueError, match="q's device"):
        F.forward_dropout(q0, k0, t((1, 1, 8, 64), 1), 0.1, 1)
    with pytest.raises(ValueError, match="workspace must be on q's device"):
        F.forward_splitkv(q0, k0, v0, num_splits=2, workspace=t((1 << 20,), 1, torch.uint8))
    q8 = t((1, 2, 8, 128), 0, torch.uint8)
    with pytest.raises(ValueError, match="q's device"):
        F.forward_fp8(q8, t((1, 1, 8, 128), 1, torch.uint8), t((1, 1, 8, 128), 0, torch.uint8),
                      1.0, 1.0, 1.0)
