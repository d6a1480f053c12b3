"""GPU parity of the tcgen05 path (128-row tensor-memory tiles) with the route
pinned, against the oracle, and agreement between the two routes."""
import pytest
import torch

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


@pytest.mark.parametrize("kind,dt", [("rising", "bf16"), ("rising", "f16"), ("falling", "bf16"),
                                     ("flat_rows", "bf16")])
def test_tc_reference_moves_inside_plain_blocks(cuda_lib, kind, dt):
    """Unmasked blocks first take P against the reference in use and take the
    row max only when the block's row sum reaches 224.  Keys whose scale
    grows along the sequence move the reference in later unmasked blocks
    (sums far above 224, with and without a move); keys whose scale shrinks
    leave every later block far below the reference (P near underflow);
    query heads of zeros give rows of equal scores, whose sums are exactly
    the block width.  All against the oracle, on the one-tile route."""
    from oracle import sdpa_oracle
    from tests.gpu_util import TOL_MAX, TOL_MEAN, compare
    p = I.Problem(1, 4, 2, 256, 2048, 128, 128, dt, False, 0, None, 31, kind)
    q, k, v = I.make_qkv(p)
    if kind in ("rising", "falling"):
        g = 1.0 + 8.0 * torch.arange(p.S, dtype=torch.float32) / p.S  # x1 .. x9
        if kind == "falling":
            g = g.flip(0)
        k = (k.float() * g[None, None, :, None]).to(k.dtype)
    else:
        q[:, ::2] = 0
    out, info = run_gpu(cuda_lib, p, q, k, v, force_path=S.PATH_TC)
    assert info["path"] == S.PATH_TC
    ref = sdpa_oracle(q, k, v, p.sm_scale, p.causal, p.window)
    mx, mean = compare(p, out.float().cpu().numpy(), ref)
    assert mx <= TOL_MAX[dt] and mean <= TOL_MEAN, f"{kind}: max {mx:.3e} mean {mean:.3e}"


@pytest.mark.parametrize("case", [
    # causal and windowed calls with one to two 256-row pair tiles per SM pair
    # take the one-SM kernel's 128-row tiles (router rule), at full size
    ("d256_causal_2k", 1, 16, 8, 2048, 2048, 256, 256, True, 0),
    ("d192_128_causal_1536", 1, 16, 16, 1536, 1536, 192, 128, True, 0),
    ("d192_128_window_1536", 1, 16, 16, 1536, 1536, 192, 128, True, 700),
], ids=lambda c: c[0])
def test_balance_rule_routes_to_one_sm_kernel(cuda_lib, case):
    name, B, Hq, Hkv, L, Sk, Dqk, Dv, causal, W = case
    p = I.Problem(B, Hq, Hkv, L, Sk, Dqk, Dv, "bf16", causal, W, None, 33, name)
    rows = I.sample_rows(L, 256, 33, window=W)
    _, _, info = check_problem(cuda_lib, p, rows=rows)
    assert info["path"] == S.PATH_TC and info["splits"] == 1, info
