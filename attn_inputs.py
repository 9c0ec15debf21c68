"""Seeded synthetic inputs shared by the oracle tests, the CUDA parity tests and
the benchmark.

This module only draws random numbers and names the workloads; it holds none
of the attention arithmetic.  Recipe: a torch CPU ``Generator`` seeded per
case draws float32 standard normals in the order Q, K, V, dO; optional data
transforms (Q scaled by 2, K shifted by +8) are applied in float32; then each
tensor is cast (round to nearest even) to the storage dtype.  The oracle and
the GPU see identical bits.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    dtype: str = "bf16"          # "bf16", "f32" or "e4m3"
    seed: int = 0
    q_mul: float = 1.0           # Q pre-multiplied in float32 before the cast
    k_add: float = 0.0           # constant added to every K element before the cast
    backward: bool = True
    n_q: int = 0                 # query rows when fewer than N (inference shapes); 0 -> N

    @property
    def Nq(self) -> int:
        return self.n_q or self.N

    @property
    def Nk(self) -> int:
        return self.N

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


def _c5() -> list:
    out = []
    k = 0
    for d in (64, 128, 256):
        for n in (512, 2048, 8192):
            for causal in (True, False):
                out.append(Workload(f"sweep_d{d}_n{n}_{'causal' if causal else 'full'}",
                                    32768 // n, 16, 16, n, d, causal, "bf16", 500 + k))
                k += 1
    out.append(Workload("sweep_adversarial_kplus8_d128_n2048_causal", 32768 // 2048, 16, 16, 2048, 128,
                        True, "bf16", 500 + k, k_add=8.0))
    return out


# The five workloads, by what they are.
SINGLE_HEAD_F32 = Workload("single_head_f32_n256_d64", 1, 1, 1, 256, 64, False, "f32", 1)
TWO_BATCH_F32 = Workload("two_batch_f32_n1024_d64", 2, 1, 1, 1024, 64, False, "f32", 2, backward=False)
TWO_BATCH_BF16 = Workload("two_batch_bf16_n1024_d64", 2, 1, 1, 1024, 64, False, "bf16", 2, backward=False)
CAUSAL_TRAIN = Workload("causal_b4_h16_n4096_d128", 4, 16, 16, 4096, 128, True, "bf16", 3)
LONG_GQA = Workload("long_gqa_b1_hq32_hkv8_n16384_d128_q2x", 1, 32, 8, 16384, 128, True, "bf16", 4, q_mul=2.0)
SWEEP = _c5()
# Inference shape (forward only, split-KV path): batch 1, 8 heads, 512 new
# query rows against a 16384-key cache, causal bottom-right aligned.
INFER_PREFILL = Workload("inference_b1_h8_nq512_nk16384_d128", 1, 8, 8, 16384, 128, True, "bf16", 6,
                         backward=False, n_q=512)

# FP8 forward: the training shape with E4M3 inputs (forward only).
FP8_CAUSAL = Workload("fp8_causal_b4_h16_n4096_d128", 4, 16, 16, 4096, 128, True, "e4m3", 7,
                      backward=False)

ALL = [SINGLE_HEAD_F32, TWO_BATCH_F32, TWO_BATCH_BF16, CAUSAL_TRAIN, LONG_GQA] + SWEEP + [INFER_PREFILL,
                                                                                        FP8_CAUSAL]
BY_NAME = {w.name: w for w in ALL}


def make(w: Workload, *, B=None, Hq=None, Hkv=None, N=None, Nq=None, Nk=None, d=None,
         seed=None, dtype=None, q_mul=None, k_add=None):
    """Draw Q, K, V, dO for workload ``w`` (optionally with shapes overridden).

    Returns a dict of contiguous CPU tensors in the storage dtype:
    q, do: [B, Hq, Nq, d]; k, v: [B, Hkv, Nk, d]."""
    B = w.B if B is None else B
    Hq = w.Hq if Hq is None else Hq
    Hkv = w.Hkv if Hkv is None else Hkv
    N = w.N if N is None else N
    Nq = (w.n_q or N) if Nq is None else Nq
    Nk = N if Nk is None else Nk
    d = w.d if d is None else d
    seed = w.seed if seed is None else seed
    dt = w.torch_dtype if dtype is None else (torch.bfloat16 if dtype == "bf16" else torch.float32)
    q_mul = w.q_mul if q_mul is None else q_mul
    k_add = w.k_add if k_add is None else k_add
    return draw(B, Hq, Hkv, Nq, Nk, d, seed, dt, q_mul, k_add)


def draw(B, Hq, Hkv, Nq, Nk, d, seed, dtype=torch.bfloat16, q_mul=1.0, k_add=0.0):
    g = torch.Generator().manual_seed(int(seed))
    q = torch.randn(B, Hq, Nq, d, generator=g, dtype=torch.float32)
    k = torch.randn(B, Hkv, Nk, d, generator=g, dtype=torch.float32)
    v = torch.randn(B, Hkv, Nk, d, generator=g, dtype=torch.float32)
    do = torch.randn(B, Hq, Nq, d, generator=g, dtype=torch.float32)
    if q_mul != 1.0:
        q = q * q_mul
    if k_add != 0.0:
        k = k + k_add
    return {name: t.to(dtype).contiguous() for name, t in (("q", q), ("k", k), ("v", v), ("do", do))}


E4M3_MAX = 448.0


def draw_fp8(B, Hq, Hkv, N, d, seed, q_mul=1.0):
    """E4M3 inputs: the float32 normals of ``draw`` for Q, K, V, each tensor
    divided by one factor (its largest magnitude / 448, rounded to float32),
    clamped to +-448 and cast by torch to float8_e4m3fn (round to nearest
    even).  Returns uint8 code tensors q, k, v and the factors descale_q,
    descale_k, descale_v (Python floats, exact float32 values)."""
    t = draw(B, Hq, Hkv, N, N, d, seed, torch.float32, q_mul)
    out = {}
    for name in ("q", "k", "v"):
        x = t[name]
        amax = float(x.abs().max())
        ds = float(torch.tensor(max(amax, 1e-30) / E4M3_MAX, dtype=torch.float32))
        codes = (x / ds).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn).view(torch.uint8)
        out[name] = codes.contiguous()
        out["descale_" + name] = ds
    return out


def make_fp8(w: Workload, *, B=None, Hq=None, Hkv=None, N=None, d=None, seed=None):
    """``draw_fp8`` for workload ``w`` (optionally with shapes overridden)."""
    return draw_fp8(w.B if B is None else B, w.Hq if Hq is None else Hq,
                    w.Hkv if Hkv is None else Hkv, w.N if N is None else N,
                    w.d if d is None else d, w.seed if seed is None else seed, w.q_mul)


def as_f64(t):
    """Exact float64 numpy copy of a float32/bf16 tensor."""
    return t.detach().to("cpu").to(torch.float64).numpy()
