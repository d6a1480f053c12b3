"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare with the fp64 oracle on the same seeded inputs.

Tolerances (written here, used by every GPU test): max |GPU - oracle| <=
2e-2 for bf16 outputs and <= 5e-3 for fp16 outputs, and mean |GPU - oracle|
<= 2e-3.  They follow from the arithmetic: inputs are exact 16-bit values,
scores and the softmax run in fp32, P is rounded to the 16-bit input type
before the P*V product (relative error 2^-8 for bf16, 2^-11 for fp16 per
weight, averaging out over many keys), and the output is rounded once
(half an ulp: up to 2^-9 relative for bf16, 2^-12 for fp16, on |O| <~ 3).
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import sdpa_oracle
from scaled_dot_product_13_b200.inputs import Problem, make_qkv

TOL_MAX = {"bf16": 2e-2, "f16": 5e-3}
TOL_MEAN = 2e-3

# GPU-vs-GPU agreement (two routes, split counts, layouts of the same
# problem).  Both results are the same softmax up to rounding order: fp32
# accumulation in another order, P rounded to 16 bits from slightly different
# exponentials (MUFU or the FMA-pipe polynomial), and one final rounding of O.
# The last step alone can flip an output by one unit in the last place of the
# output type, i.e. up to 2^-7 (bf16) / 2^-10 (fp16) of its magnitude, so
# the bound is an absolute part plus one such unit.
AGREE_ABS = {"bf16": 4e-3, "f16": 1e-3}
AGREE_ULP = {"bf16": 2.0 ** -7, "f16": 2.0 ** -10}


def agree(a, b, dtype: str) -> bool:
    """True when |a - b| <= AGREE_ABS + one output ulp of |b|, elementwise."""
    a = a.float()
    b = b.float()
    return bool(((a - b).abs() <= AGREE_ABS[dtype] + AGREE_ULP[dtype] * b.abs()).all())


def run_gpu(sdpa, p: Problem, q, k, v, force_path=0, force_splits=0, guard=True):
    """Run one call with an explicit workspace and canary guard bands around
    the output; returns the output (CUDA tensor) after checking the canaries."""
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    info = sdpa.plan(p.B, p.Hq, p.Hkv, p.L, p.S, p.Dqk, p.Dv, p.causal, p.window, p.dtype,
                     force_path=force_path, force_splits=force_splits)
    n_out = p.B * p.Hq * p.L * p.Dv
    pad = 4096
    buf = torch.full((n_out + 2 * pad,), 1234.5, dtype=q.dtype, device="cuda")
    out = buf[pad:pad + n_out].view(p.B, p.Hq, p.L, p.Dv)
    ws_bytes = info["workspace_bytes"]
    ws = None
    if ws_bytes:
        ws_buf = torch.full((ws_bytes // 4 + 2 * pad,), 7.25, dtype=torch.float32, device="cuda")
        ws = ws_buf[pad:pad + ws_bytes // 4]
    sdpa.forward_ws(qd, kd, vd, ws, scale=p.sm_scale, causal=p.causal, window_size=p.window,
                    out=out, force_path=force_path, force_splits=force_splits)
    sdpa.device_status(clear=True)
    if guard:
        assert torch.all(buf[:pad] == 1234.5) and torch.all(buf[pad + n_out:] == 1234.5), \
            "output guard band overwritten"
        if ws is not None:
            assert torch.all(ws_buf[:pad] == 7.25) and torch.all(ws_buf[pad + ws_bytes // 4:] == 7.25), \
                "workspace guard band overwritten"
    return out, info


def compare(p: Problem, got, ref):
    got = got.astype(np.float64)
    assert np.all(np.isfinite(got)), "non-finite output"
    err = np.abs(got - ref)
    return float(err.max()), float(err.mean())


def check_problem(sdpa, p: Problem, rows=None, force_path=0, force_splits=0, seed=None):
    q, k, v = make_qkv(p, seed)
    out, info = run_gpu(sdpa, p, q, k, v, force_path, force_splits)
    got = out.float().cpu().numpy()
    if rows is not None:
        got = got[:, :, rows]
    ref = sdpa_oracle(q, k, v, p.sm_scale, p.causal, p.window, rows=rows)
    mx, mean = compare(p, got, ref)
    assert mx <= TOL_MAX[p.dtype] and mean <= TOL_MEAN, \
        f"{p.name or p}: max abs {mx:.3e} mean abs {mean:.3e} (plan {info})"
    return mx, mean, info
