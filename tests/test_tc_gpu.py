"""GPU parity of the tcgen05 path (128-row tensor-memory tiles) with the route
pinned, against the oracle, and agreement between the two routes."""
import pytest

import scaled_dot_product_13_b200 as S
from scaled_dot_product_13_b200 import inputs as I
from tests.gpu_util import agree, check_problem, run_gpu

pytestmark = pytest.mark.gpu

CASES = [
    # name, B, Hq, Hkv, L, S, Dqk, Dv, dtype, causal, window
    ("tc_d64_one_tile", 1, 1, 1, 128, 128, 64, 64, "bf16", False, 0),
    ("tc_d64_causal", 1, 2, 1, 256, 256, 64, 64, "bf16", True, 0),
    ("tc_d128_ragged", 1, 2, 2, 200, 333, 128, 128, "f16", False, 0),
    ("tc_d128_causal_gqa", 2, 4, 2, 300, 300, 128, 128, "bf16", True, 0),
    ("tc_d72", 1, 2, 2, 257, 257, 72, 72, "bf16", False, 0),
    ("tc_d192_128", 1, 2, 1, 130, 500, 192, 128, "bf16", True, 0),
    ("tc_d192", 1, 2, 2, 140, 140, 192, 192, "f16", True, 0),
    ("tc_d256_window", 1, 4, 2, 400, 400, 256, 256, "bf16", True, 100),
    ("tc_d256_window_lt_s", 1, 2, 1, 150, 700, 256, 256, "bf16", True, 200),
    ("tc_verify_packed", 1, 32, 8, 32, 2000, 128, 128, "f16", False, 0),
    ("tc_verify_packed_l64", 1, 32, 8, 64, 3000, 128, 128, "f16", True, 0),
    ("tc_l_gt_s", 1, 2, 2, 160, 40, 64, 64, "bf16", False, 0),
    ("tc_small_dims", 1, 2, 1, 130, 90, 32, 48, "bf16", False, 0),
    ("tc_window_1", 1, 2, 1, 140, 140, 64, 64, "bf16", True, 1),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_tc_vs_oracle(cuda_lib, case):
    name, B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W = case
    p = I.Problem(B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W, None, 21, name)
    _, _, info = check_problem(cuda_lib, p, force_path=S.PATH_TC)
    assert info["path"] == S.PATH_TC


@pytest.mark.parametrize("scale", [-0.09, 0.0, 0.5])
@pytest.mark.parametrize("path", [S.PATH_TC, S.PATH_SPLITKV])
def test_unusual_scales(cuda_lib, scale, path):
    # a negative scale flips which score is the row max; zero gives uniform
    # weights over the visible keys
    p = I.Problem(1, 4, 2, 150, 260, 128, 128, "bf16", True, 30, scale, 24, "scales")
    check_problem(cuda_lib, p, force_path=path)


@pytest.mark.parametrize("splits", [2, 5, 0])
def test_tc_with_key_splits(cuda_lib, splits):
    p = I.Problem(1, 8, 2, 64, 3000, 128, 128, "bf16", True, 0, None, 22, "tc_split")
    _, _, info = check_problem(cuda_lib, p, force_path=S.PATH_TC, force_splits=splits)
    assert info["path"] == S.PATH_TC


@pytest.mark.parametrize("case", CASES[:10], ids=[c[0] for c in CASES[:10]])
def test_routes_agree(cuda_lib, case):
    name, B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W = case
    p = I.Problem(B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W, None, 23, name)
    q, k, v = I.make_qkv(p)
    a = run_gpu(cuda_lib, p, q, k, v, force_path=S.PATH_TC)[0].float()
    b = run_gpu(cuda_lib, p, q, k, v, force_path=S.PATH_SPLITKV)[0].float()
    assert agree(a, b, dt)
