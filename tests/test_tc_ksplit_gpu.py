"""GPU parity of the key-split tcgen05 path (one 128-row tile per CTA whose two
softmax groups take alternate key blocks and are merged in the epilogue)
against the oracle, and agreement with the one-tile path.  Key ranges of 0,
1, 2 and 3 blocks per CTA cover a group with no block, with one block each,
and an odd split of the blocks."""
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
    ("one_block", 1, 2, 2, 100, 100, 64, 64, "bf16", True, 0),
    ("two_blocks", 1, 2, 2, 128, 256, 64, 64, "bf16", False, 0),
    ("three_blocks_ragged", 1, 2, 1, 77, 301, 128, 128, "f16", False, 0),
    ("d64_causal_gqa", 1, 8, 2, 300, 600, 64, 64, "bf16", True, 0),
    ("d72_ragged", 1, 3, 3, 333, 371, 72, 72, "bf16", False, 0),
    ("d80_f16_causal", 2, 8, 2, 200, 260, 80, 80, "f16", True, 0),
    ("d128_window", 1, 4, 2, 700, 700, 128, 128, "bf16", True, 150),
    ("d128_window_1", 1, 2, 1, 300, 300, 128, 128, "f16", True, 1),
    ("d40_24", 1, 2, 1, 300, 333, 40, 24, "bf16", False, 0),
    ("verify_like", 1, 32, 8, 24, 5000, 128, 128, "f16", False, 0),
    ("d128_noncausal_l_gt_s", 1, 2, 2, 400, 150, 128, 128, "bf16", False, 0),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_tc_ksplit_vs_oracle(cuda_lib, case):
    name, B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W = case
    p = I.Problem(B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W, None, 71, name)
    _, _, info = check_problem(cuda_lib, p, force_path=S.PATH_TC_KSPLIT)
    assert info["path"] == S.PATH_TC_KSPLIT and info["row_tile"] == 128


@pytest.mark.parametrize("splits", [2, 3, 7, 0])
def test_tc_ksplit_key_splits(cuda_lib, splits):
    # 7 splits of 4000 keys: some splits hold one or two blocks
    p = I.Problem(1, 8, 2, 32, 4000, 128, 128, "f16", False, 0, None, 72, "ksplit_split")
    _, _, info = check_problem(cuda_lib, p, force_path=S.PATH_TC_KSPLIT, force_splits=splits)
    assert info["path"] == S.PATH_TC_KSPLIT


def test_tc_ksplit_sinks_offset_lse(cuda_lib):
    p = I.Problem(1, 4, 2, 300, 900, 64, 64, "bf16", True, 250, None, 73, "ksplit_ex")
    q, k, v = I.make_qkv(p)
    sinks = [0.5, -1.0, 2.0, 0.0]
    for fs in (1, 3):
        lse = torch.full((1, 4, 300), float("nan"), dtype=torch.float32, device="cuda")
        out = cuda_lib.forward_ex(q.cuda(), k.cuda(), v.cuda(), scale=p.sm_scale, causal=True,
                                  window_size=250, q_offset=500,
                                  sinks=torch.tensor(sinks, device="cuda"), lse=lse,
                                  force_path=S.PATH_TC_KSPLIT, force_splits=fs)
        cuda_lib.device_status()
        ref, ref_lse = sdpa_oracle(q, k, v, p.sm_scale, True, 250, q_offset=500, sinks=sinks,
                                   return_lse=True)
        err = np.abs(out.float().cpu().numpy() - ref)
        assert err.max() <= TOL_MAX["bf16"] and err.mean() <= TOL_MEAN
        assert np.abs(lse.cpu().numpy() - ref_lse).max() <= 2e-3


@pytest.mark.parametrize("case", CASES[3:8], ids=[c[0] for c in CASES[3:8]])
def test_tc_ksplit_agrees_with_tc(cuda_lib, case):
    name, B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W = case
    p = I.Problem(B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W, None, 74, name)
    q, k, v = I.make_qkv(p)
    a = run_gpu(cuda_lib, p, q, k, v, force_path=S.PATH_TC_KSPLIT)[0].float()
    b = run_gpu(cuda_lib, p, q, k, v, force_path=S.PATH_TC)[0].float()
    assert agree(a, b, dt)


@pytest.mark.parametrize("scale", [-0.09, 0.0, 0.5])
def test_tc_ksplit_unusual_scales(cuda_lib, scale):
    p = I.Problem(1, 4, 2, 300, 420, 64, 64, "bf16", True, 0, scale, 75, "ksplit_scales")
    check_problem(cuda_lib, p, force_path=S.PATH_TC_KSPLIT)
