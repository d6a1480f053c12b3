"""Seeded synthetic inputs and the benchmark shapes.

This module only draws random numbers and names shapes; it holds none of the
attention arithmetic.  Both the CUDA path (tests, bench, smoke) and the CPU
oracle read the same tensors from here.

Recipe: Q, K and V are drawn i.i.d. N(0, 1) in fp32 from
``torch.Generator('cpu').manual_seed(seed)`` in the order q, k, v, then cast
(round to nearest even) to the 16-bit input type.  The oracle reads the cast
values exactly (bf16/fp16 -> fp64 is exact).  The pages draw from
``mx.random.normal`` with no seed (mlx issue #3826, repro); the seeding is
ours.

The shapes stand in for the model layers the pages measure (an audio
encoder, a vision encoder with head dim 72, MiMo-style asymmetric 192/128
decode, a GQA 32/8 verify sweep, Gemma-style 256-wide sliding-window
layers); no model weights or datasets are involved.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Problem:
    B: int
    Hq: int
    Hkv: int
    L: int
    S: int
    Dqk: int
    Dv: int
    dtype: str  # "bf16" | "f16"
    causal: bool
    window: int = 0
    scale: float | None = None  # None -> Dqk ** -0.5
    seed: int = 0
    name: str = ""

    @property
    def sm_scale(self) -> float:
        return self.scale if self.scale is not None else self.Dqk ** -0.5

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float16

    def with_(self, **kw) -> "Problem":
        return dataclasses.replace(self, **kw)


def make_qkv(p: Problem, seed: int | None = None):
    """Return (q, k, v) CPU tensors of ``p.torch_dtype`` in [B, H, N, D] layout."""
    g = torch.Generator("cpu").manual_seed(p.seed if seed is None else seed)
    dt = p.torch_dtype
    q = torch.randn(p.B, p.Hq, p.L, p.Dqk, generator=g, dtype=torch.float32).to(dt)
    k = torch.randn(p.B, p.Hkv, p.S, p.Dqk, generator=g, dtype=torch.float32).to(dt)
    v = torch.randn(p.B, p.Hkv, p.S, p.Dv, generator=g, dtype=torch.float32).to(dt)
    return q, k, v


def sample_rows(L: int, n: int = 256, seed: int = 0, window: int = 0, block: int = 128):
    """Seeded sample of query rows for the large problems.

    Always holds row 0, row L-1, the rows on both sides of every ``block``
    boundary and of the window edge (L - window), and fills up to ``n`` rows
    with uniform draws from ``numpy.random.default_rng(seed + 1000)``.
    """
    if L <= n:
        return list(range(L))
    must = {0, L - 1}
    for e in range(block, L, block):
        must.update({e - 1, e})
    if window and 0 < L - window < L:
        must.update({L - window - 1, L - window, L - window + 1})
    must = sorted(r for r in must if 0 <= r < L)
    if len(must) > n // 2:  # keep room for the uniform draws
        idx = np.linspace(0, len(must) - 1, n // 2).round().astype(int)
        must = sorted({must[i] for i in idx} | {0, L - 1})
    rng = np.random.default_rng(seed + 1000)
    pool = np.setdiff1d(np.arange(L), np.asarray(must))
    extra = rng.choice(pool, size=min(n - len(must), pool.size), replace=False)
    return sorted(set(must) | set(int(x) for x in extra))


# --- the five workloads -------------------------------------------------------

def tiny_problem() -> Problem:
    """Tiny causal GQA prefill, the small case the oracle finishes instantly."""
    return Problem(1, 4, 2, 128, 128, 64, 64, "bf16", True, 0, 1.0 / 8.0, 0, "tiny_causal_gqa")


DECODE_S = (256, 1024, 4096, 8192, 16384, 32768)


def decode_problems():
    """Decode, L=1, Hq=64, Hkv in {4, 8}, Dqk=192/Dv=128, bf16, causal."""
    out = []
    for hkv in (4, 8):
        for s in DECODE_S:
            out.append(Problem(1, 64, hkv, 1, s, 192, 128, "bf16", True, 0,
                               192 ** -0.5, 1, f"decode_hkv{hkv}_s{s}"))
    return out


VERIFY_L = (1, 2, 4, 8, 12, 16, 24, 32, 48, 64)


def verify_problems(S_list=(16384, 32768), L_list=VERIFY_L):
    """Verify sweep, GQA 32/8, D=128, fp16, no mask."""
    return [Problem(1, 32, 8, L, S, 128, 128, "f16", False, 0, 128 ** -0.5, 2,
                    f"verify_s{S}_l{L}") for S in S_list for L in L_list]


def encoder_problems():
    """Non-causal encoder prefill: D=64 at 1500 tokens, D=72 at 1024/4096."""
    return [Problem(1, 20, 20, 1500, 1500, 64, 64, "bf16", False, 0, None, 3, "encoder_h20_l1500_d64"),
            Problem(1, 16, 16, 1024, 1024, 72, 72, "bf16", False, 0, None, 3, "encoder_h16_l1024_d72"),
            Problem(1, 16, 16, 4096, 4096, 72, 72, "bf16", False, 0, None, 3, "encoder_h16_l4096_d72")]


def window_problems(include_32k: bool = True):
    """Sliding-window causal prefill, D=256, W=1024; plus full causal 32K."""
    out = [Problem(1, 16, 8, n, n, 256, 256, "bf16", True, 1024, None, 4, f"window_l{n}_w1024_d256")
           for n in (2048, 4096, 8192)]
    if include_32k:
        out.append(Problem(1, 16, 8, 32768, 32768, 256, 256, "bf16", True, 0, None, 4,
                           "causal_l32768_d256"))
    return out


def wide_problems():
    """Head dim 512: decode (16 query heads on one KV head) at 8K and 32K keys,
    and a causal prefill of 4096 tokens over 8 heads.  The pages name head dim
    512 as the case their fused kernels do not cover; no page measures it, so
    these shapes extend the decode and prefill workloads above."""
    out = [Problem(1, 16, 1, 1, s, 512, 512, "bf16", True, 0, None, 5, f"wide_decode_d512_s{s}")
           for s in (8192, 32768)]
    out.append(Problem(1, 8, 8, 4096, 4096, 512, 512, "bf16", True, 0, None, 5,
                       "wide_prefill_d512_l4096"))
    return out


__all__ = ["Problem", "make_qkv", "sample_rows", "tiny_problem", "decode_problems",
           "verify_problems", "encoder_problems", "window_problems", "wide_problems",
           "DECODE_S", "VERIFY_L"]
