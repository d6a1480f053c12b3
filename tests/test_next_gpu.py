"""GPU parity of sdpa_forward_ex: explicit query offset (chunked prefill,
rotating window cache), attention sinks and the LSE output, on both routes
and with split keys, against the fp64 oracle."""
import numpy as np
import pytest
import torch

import scaled_dot_product_13_b200 as S
from oracle import sdpa_oracle
from scaled_dot_product_13_b200 import inputs as I
from tests.gpu_util import TOL_MAX, TOL_MEAN

pytestmark = pytest.mark.gpu

LSE_TOL = 2e-3  # fp32 scores and sums; only O carries the 16-bit rounding of P


def _run(sdpa, p, q, k, v, q_offset=None, sinks=None, path=0, splits=0):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    lse = torch.full((p.B, p.Hq, p.L), float("nan"), dtype=torch.float32, device="cuda")
    sk = None if sinks is None else torch.tensor(sinks, dtype=torch.float32, device="cuda")
    out = sdpa.forward_ex(qd, kd, vd, scale=p.sm_scale, causal=p.causal, window_size=p.window,
                          q_offset=q_offset, sinks=sk, lse=lse, force_path=path,
                          force_splits=splits)
    sdpa.device_status()
    return out.float().cpu().numpy(), lse.cpu().numpy()


def _check(p, got, lse, ref, ref_lse):
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)) and err.max() <= TOL_MAX[p.dtype] and err.mean() <= TOL_MEAN, \
        f"max {err.max():.3e} mean {err.mean():.3e}"
    lerr = np.abs(lse - ref_lse)
    assert np.all(np.isfinite(lse)) and lerr.max() <= LSE_TOL, f"lse err {lerr.max():.3e}"


PATHS = [(S.PATH_TC, 0), (S.PATH_SPLITKV, 0), (S.PATH_SPLITKV, 5), (S.PATH_TC, 3)]


@pytest.mark.parametrize("path,splits", PATHS)
@pytest.mark.parametrize("W", [0, 90])
def test_chunked_prefill(cuda_lib, path, splits, W):
    N, c0, c1 = 700, 256, 520
    full = I.Problem(1, 4, 2, N, N, 128, 128, "bf16", True, W, None, 31, "chunk")
    q, k, v = I.make_qkv(full)
    p = full.with_(L=c1 - c0, S=c1)
    qc, kc, vc = q[:, :, c0:c1].contiguous(), k[:, :, :c1].contiguous(), v[:, :, :c1].contiguous()
    got, lse = _run(cuda_lib, p, qc, kc, vc, q_offset=c0, path=path, splits=splits)
    ref, ref_lse = sdpa_oracle(qc, kc, vc, p.sm_scale, True, W, q_offset=c0, return_lse=True)
    _check(p, got, lse, ref, ref_lse)
    # the same rows of the full causal prefill
    ref_full = sdpa_oracle(q, k, v, full.sm_scale, True, W)[:, :, c0:c1]
    assert np.abs(ref - ref_full).max() < 1e-12


@pytest.mark.parametrize("path,splits", PATHS)
def test_rotating_window_cache(cuda_lib, path, splits):
    # the cache holds the last W + L - 1 keys; positions are relative to it
    W, L = 128, 40
    p = I.Problem(1, 8, 2, L, W + L - 1, 64, 64, "f16", True, W, None, 32, "rotating")
    q, k, v = I.make_qkv(p)
    got, lse = _run(cuda_lib, p, q, k, v, q_offset=W - 1, path=path, splits=splits)
    ref, ref_lse = sdpa_oracle(q, k, v, p.sm_scale, True, W, q_offset=W - 1, return_lse=True)
    _check(p, got, lse, ref, ref_lse)


@pytest.mark.parametrize("path,splits", PATHS)
@pytest.mark.parametrize("causal", [True, False])
def test_sinks(cuda_lib, path, splits, causal):
    p = I.Problem(1, 8, 2, 150, 400, 128, 128, "bf16", causal, 0, None, 33, "sinks")
    q, k, v = I.make_qkv(p)
    sinks = list(np.random.default_rng(3).uniform(-2, 4, size=8))
    got, lse = _run(cuda_lib, p, q, k, v, sinks=sinks, path=path, splits=splits)
    ref, ref_lse = sdpa_oracle(q, k, v, p.sm_scale, causal, 0, sinks=sinks, return_lse=True)
    _check(p, got, lse, ref, ref_lse)


def test_decode_with_sinks_and_lse(cuda_lib):
    p = I.decode_problems()[4]  # Hkv=4, S=16384: split keys + combine
    q, k, v = I.make_qkv(p)
    sinks = list(np.linspace(-1, 3, p.Hq))
    got, lse = _run(cuda_lib, p, q, k, v, sinks=sinks)
    ref, ref_lse = sdpa_oracle(q, k, v, p.sm_scale, True, 0, sinks=sinks, return_lse=True)
    _check(p, got, lse, ref, ref_lse)


def test_lse_plain_configs(cuda_lib):
    for p in (I.tiny_problem(), I.verify_problems(S_list=(16384,), L_list=(12, 64))[0],
              I.verify_problems(S_list=(16384,), L_list=(12, 64))[1]):
        q, k, v = I.make_qkv(p)
        got, lse = _run(cuda_lib, p, q, k, v)
        ref, ref_lse = sdpa_oracle(q, k, v, p.sm_scale, p.causal, p.window, return_lse=True)
        _check(p, got, lse, ref, ref_lse)


def test_offset_errors(cuda_lib):
    q = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 2, 16, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cuda_lib.SdpaError) as ei:
        cuda_lib.forward_ex(q, k, k, causal=True, q_offset=-1)
    assert "q_offset >= 0" in ei.value.message
    with pytest.raises(cuda_lib.SdpaError) as ei:
        cuda_lib.forward_ex(q, k, k, causal=True, window_size=4, q_offset=30)
    assert "sees no key" in ei.value.message
