"""GPU parity of the two-CTA path (tcgen05 cta_group::2 over 256-row tiles
shared by a pair of SMs) against the oracle, and agreement with the one-CTA
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
    ("d256_one_pair", 1, 1, 1, 256, 256, 256, 256, "bf16", False, 0),
    ("d256_causal", 1, 2, 1, 512, 512, 256, 256, "bf16", True, 0),
    ("d256_ragged", 1, 2, 2, 300, 333, 256, 256, "f16", False, 0),
    ("d256_window", 1, 4, 2, 700, 700, 256, 256, "bf16", True, 150),
    ("d256_window_lt_s", 1, 2, 1, 200, 900, 256, 256, "bf16", True, 300),
    ("d256_gqa_half_pair", 1, 2, 1, 130, 260, 256, 256, "bf16", True, 0),
    ("d192_128", 1, 4, 1, 140, 500, 192, 128, "bf16", True, 0),
    ("d192_128_f16", 2, 2, 2, 400, 400, 192, 128, "f16", False, 0),
    ("d256_small_pair_rows", 1, 1, 1, 64, 64, 256, 256, "bf16", True, 0),
    ("d256_window_1", 1, 2, 1, 260, 260, 256, 256, "bf16", True, 1),
    ("d128_causal", 1, 4, 2, 600, 600, 128, 128, "bf16", True, 0),
    ("d128_f16_window", 2, 4, 4, 300, 450, 128, 128, "f16", True, 77),
    ("d64_padded", 1, 4, 4, 512, 512, 64, 64, "bf16", False, 0),
    ("d72_padded", 1, 2, 2, 700, 700, 72, 72, "bf16", False, 0),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_tc2_vs_oracle(cuda_lib, case):
    name, B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W = case
    p = I.Problem(B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W, None, 41, name)
    _, _, info = check_problem(cuda_lib, p, force_path=S.PATH_TC2)
    assert info["path"] == S.PATH_TC2


@pytest.mark.parametrize("splits", [2, 7, 0])
def test_tc2_with_key_splits(cuda_lib, splits):
    p = I.Problem(1, 4, 2, 256, 3000, 256, 256, "bf16", True, 0, None, 42, "tc2_split")
    _, _, info = check_problem(cuda_lib, p, force_path=S.PATH_TC2, force_splits=splits)
    assert info["path"] == S.PATH_TC2


def test_tc2_sinks_offset_lse(cuda_lib):
    p = I.Problem(1, 4, 2, 300, 800, 256, 256, "bf16", True, 200, None, 43, "tc2_ex")
    q, k, v = I.make_qkv(p)
    sinks = [0.5, -1.0, 2.0, 0.0]
    lse = torch.full((1, 4, 300), float("nan"), dtype=torch.float32, device="cuda")
    out = cuda_lib.forward_ex(q.cuda(), k.cuda(), v.cuda(), scale=p.sm_scale, causal=True,
                              window_size=200, q_offset=450,
                              sinks=torch.tensor(sinks, device="cuda"), lse=lse,
                              force_path=S.PATH_TC2)
    cuda_lib.device_status()
    ref, ref_lse = sdpa_oracle(q, k, v, p.sm_scale, True, 200, q_offset=450, sinks=sinks,
                               return_lse=True)
    err = np.abs(out.float().cpu().numpy() - ref)
    assert err.max() <= TOL_MAX["bf16"] and err.mean() <= TOL_MEAN
    assert np.abs(lse.cpu().numpy() - ref_lse).max() <= 2e-3


@pytest.mark.parametrize("case", CASES[:6], ids=[c[0] for c in CASES[:6]])
def test_tc2_agrees_with_tc(cuda_lib, case):
    name, B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W = case
    p = I.Problem(B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W, None, 44, name)
    q, k, v = I.make_qkv(p)
    a = run_gpu(cuda_lib, p, q, k, v, force_path=S.PATH_TC2)[0].float()
    b = run_gpu(cuda_lib, p, q, k, v, force_path=S.PATH_TC)[0].float()
    assert agree(a, b, dt)


# More 256-row tiles than SM pairs (several waves of CTA pairs), mixed tile
# weights; with causal masking and forced key splits some (tile, split) units
# see no key block at all.
WALK = [
    # name, B, Hq, Hkv, L, S, causal, window, force_splits
    ("walk_causal", 2, 16, 16, 1024, 1024, True, 0, 0),
    ("walk_gqa_noncausal", 3, 32, 8, 512, 640, False, 0, 0),
    ("walk_window", 2, 16, 8, 1536, 1536, True, 200, 0),
    ("walk_split_empty_items", 2, 16, 16, 1024, 1024, True, 0, 3),
]


@pytest.mark.parametrize("case", WALK, ids=[c[0] for c in WALK])
def test_tc2_many_waves(cuda_lib, case):
    name, B, Hq, Hkv, L, Sk, causal, W, fs = case
    p = I.Problem(B, Hq, Hkv, L, Sk, 256, 256, "bf16", causal, W, None, 45, name)
    rows = sorted(set([0, 1, 127, 128, 255, 256, L // 2, L - 129, L - 2, L - 1]))
    _, _, info = check_problem(cuda_lib, p, rows=rows, force_path=S.PATH_TC2, force_splits=fs)
    assert info["path"] == S.PATH_TC2
    assert info["ctas"] > 74


@pytest.mark.parametrize("scale", [-0.05, 0.0, 0.3])
def test_tc2_unusual_scales(cuda_lib, scale):
    p = I.Problem(1, 4, 2, 300, 450, 256, 256, "bf16", True, 100, scale, 46, "tc2_scales")
    check_problem(cuda_lib, p, force_path=S.PATH_TC2)
