"""GPU parity of the two-tile tcgen05 path (two 128-row query tiles per CTA
sharing every K/V block) against the oracle, and agreement with the one-tile
path."""
import numpy as np
import pytest
import torch

import scaled_dot_product_13_b200 as S
from oracle import sdpa_oracle
from scaled_dot_product_13_b200 import inputs as I
from tests.gpu_util import agree, TOL_MAX, TOL_MEAN, check_problem, run_gpu

pytestmark = pytest.mark.gpu

CASES = [
    # name, B, Hq, Hkv, L, S, Dqk, Dv, dtype, causal, window
    ("d64_one_tile_pair", 1, 2, 2, 256, 256, 64, 64, "bf16", False, 0),
    ("d64_causal", 1, 4, 2, 600, 600, 64, 64, "bf16", True, 0),
    ("d64_half_pair", 1, 1, 1, 130, 300, 64, 64, "bf16", True, 0),
    ("d72_ragged", 1, 3, 3, 333, 371, 72, 72, "bf16", False, 0),
    ("d80_f16_causal_gqa", 2, 8, 2, 200, 260, 80, 80, "f16", True, 0),
    ("d72_window", 1, 4, 2, 500, 500, 72, 72, "bf16", True, 100),
    ("d72_causal_long", 1, 2, 2, 1000, 2000, 72, 72, "bf16", True, 0),
    ("d128_window", 1, 4, 2, 700, 700, 128, 128, "bf16", True, 150),
    ("d128_window_1", 1, 2, 1, 300, 300, 128, 128, "f16", True, 1),
    ("d128_l_lt_s", 1, 4, 4, 257, 1000, 128, 128, "bf16", True, 0),
    ("d40_24", 1, 2, 1, 300, 333, 40, 24, "bf16", False, 0),
    ("d128_noncausal_l_gt_s", 1, 2, 2, 400, 150, 128, 128, "bf16", False, 0),
    ("encoder_like_d64", 1, 20, 20, 1500, 1500, 64, 64, "bf16", False, 0),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_tc_dual_vs_oracle(cuda_lib, case):
    name, B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W = case
    p = I.Problem(B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W, None, 61, name)
    rows = I.sample_rows(L, 256, seed=61) if L > 1024 else None
    _, _, info = check_problem(cuda_lib, p, rows=rows, force_path=S.PATH_TC_DUAL)
    assert info["path"] == S.PATH_TC_DUAL and info["row_tile"] == 256


@pytest.mark.parametrize("splits", [2, 5, 0])
def test_tc_dual_key_splits(cuda_lib, splits):
    p = I.Problem(1, 8, 2, 128, 4000, 128, 128, "f16", False, 0, None, 62, "dual_split")
    _, _, info = check_problem(cuda_lib, p, force_path=S.PATH_TC_DUAL, force_splits=splits)
    assert info["path"] == S.PATH_TC_DUAL


def test_tc_dual_sinks_offset_lse(cuda_lib):
    p = I.Problem(1, 4, 2, 300, 900, 64, 64, "bf16", True, 250, None, 63, "dual_ex")
    q, k, v = I.make_qkv(p)
    sinks = [0.5, -1.0, 2.0, 0.0]
    for fs in (1, 3):
        lse = torch.full((1, 4, 300), float("nan"), dtype=torch.float32, device="cuda")
        out = cuda_lib.forward_ex(q.cuda(), k.cuda(), v.cuda(), scale=p.sm_scale, causal=True,
                                  window_size=250, q_offset=500,
                                  sinks=torch.tensor(sinks, device="cuda"), lse=lse,
                                  force_path=S.PATH_TC_DUAL, force_splits=fs)
        cuda_lib.device_status()
        ref, ref_lse = sdpa_oracle(q, k, v, p.sm_scale, True, 250, q_offset=500, sinks=sinks,
                                   return_lse=True)
        err = np.abs(out.float().cpu().numpy() - ref)
        assert err.max() <= TOL_MAX["bf16"] and err.mean() <= TOL_MEAN
        assert np.abs(lse.cpu().numpy() - ref_lse).max() <= 2e-3


@pytest.mark.parametrize("case", CASES[:6], ids=[c[0] for c in CASES[:6]])
def test_tc_dual_agrees_with_tc(cuda_lib, case):
    name, B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W = case
    p = I.Problem(B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W, None, 64, name)
    q, k, v = I.make_qkv(p)
    a = run_gpu(cuda_lib, p, q, k, v, force_path=S.PATH_TC_DUAL)[0].float()
    b = run_gpu(cuda_lib, p, q, k, v, force_path=S.PATH_TC)[0].float()
    assert agree(a, b, dt)


@pytest.mark.parametrize("scale", [-0.09, 0.0, 0.5])
def test_tc_dual_unusual_scales(cuda_lib, scale):
    # a negative scale flips which score is the row max; zero weighs every
    # visible key the same (masked keys must still get weight 0, not NaN)
    p = I.Problem(1, 4, 2, 300, 420, 64, 64, "bf16", True, 0, scale, 65, "dual_scales")
    check_problem(cuda_lib, p, force_path=S.PATH_TC_DUAL)
