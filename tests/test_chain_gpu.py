"""Back-to-back calls whose inputs are the previous call's output (GPU).

The split pass is launched as a programmatic dependent of the kernel before
it on the stream, and prefetches its first inputs into L2 before waiting for
that kernel.  These tests chain calls so that each call's q is the previous
call's out, enqueued without any synchronisation in between (eagerly, from
one CUDA graph, and through the no-allocation entry point, whose split
partials share one scratch array): every output must match the fp64 oracle
evaluated on the previous output's actual values.  A read of q before the
previous combine finished, or partials overwritten while the previous combine
still read them, would break the match.
"""
import numpy as np
import pytest
import torch

from oracle import sdpa_oracle
from scaled_dot_product_13_b200 import inputs as I
from tests.gpu_util import TOL_MAX, TOL_MEAN, compare

pytestmark = pytest.mark.gpu

# L=1 decode shape whose output can feed the next call's q (Dqk == Dv), split
# over the keys (so every call is a split pass plus a combine)
P = I.Problem(1, 16, 4, 1, 4096, 128, 128, "bf16", False, 0, 128 ** -0.5, 11, "chain")
STEPS = 6


def _check_chain(p, q0, k, v, outs):
    prev = q0.cpu()
    kc, vc = k.cpu(), v.cpu()
    for n, out in enumerate(outs):
        ref = sdpa_oracle(prev, kc, vc, p.sm_scale, p.causal, p.window)
        mx, mean = compare(p, out.float().cpu().numpy(), ref)
        assert mx <= TOL_MAX[p.dtype] and mean <= TOL_MEAN, f"step {n}: max {mx:.3e} mean {mean:.3e}"
        prev = out.cpu()


def _inputs():
    q, k, v = I.make_qkv(P)
    # scale q up so the chained outputs keep a spread of scores
    return (q * 4).to(q.dtype).cuda(), k.cuda(), v.cuda()


def test_plan_is_split(cuda_lib):
    info = cuda_lib.plan(P.B, P.Hq, P.Hkv, P.L, P.S, P.Dqk, P.Dv, P.causal, P.window, P.dtype)
    assert info["path"] == cuda_lib.PATH_SPLITKV and info["splits"] > 1


def test_chained_calls_eager(cuda_lib):
    q0, k, v = _inputs()
    outs = [torch.full_like(q0, float("nan")) for _ in range(STEPS)]
    x = q0
    for o in outs:
        cuda_lib.forward(x, k, v, scale=P.sm_scale, out=o)
        x = o
    torch.cuda.synchronize()
    cuda_lib.device_status()
    _check_chain(P, q0, k, v, outs)


def test_chained_calls_in_one_graph(cuda_lib):
    q0, k, v = _inputs()
    info = cuda_lib.plan(P.B, P.Hq, P.Hkv, P.L, P.S, P.Dqk, P.Dv, P.causal, P.window, P.dtype)
    wss = [torch.empty(info["workspace_bytes"] // 4, dtype=torch.float32, device="cuda")
           for _ in range(STEPS)]
    outs = [torch.empty_like(q0) for _ in range(STEPS)]

    def body():
        x = q0
        for o, ws in zip(outs, wss):
            cuda_lib.forward_ws(x, k, v, ws, scale=P.sm_scale, out=o)
            x = o

    body()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        body()
    for o in outs:
        o.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    cuda_lib.device_status()
    _check_chain(P, q0, k, v, outs)
    del g


def test_chained_calls_share_the_noalloc_scratch(cuda_lib):
    q0, k, v = _inputs()
    outs = [torch.full_like(q0, float("nan")) for _ in range(STEPS)]
    x = q0
    for o in outs:
        cuda_lib.forward_noalloc(x, k, v, scale=P.sm_scale, out=o)
        x = o
    torch.cuda.synchronize()
    cuda_lib.device_status()
    _check_chain(P, q0, k, v, outs)
