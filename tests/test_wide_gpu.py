"""GPU parity at head dims above 256 (up to 512) against the oracle: the wide
path (the output columns split over four warps per 16-row group), the
tcgen05 path in column halves (one CTA per 256-column half of V and O, each
computing the full scores) and the pair kernel in column halves (an SM pair
per 256-row tile and 256-column half, 64-key blocks)."""
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
    ("decode_g16_s1", 1, 16, 1, 1, 1, 512, 512, "bf16", True, 0),
    ("decode_g16_s33", 1, 16, 1, 1, 33, 512, 512, "bf16", True, 0),
    ("decode_g16_s4096", 1, 16, 1, 1, 4096, 512, 512, "bf16", True, 0),
    ("decode_g8_s20000", 2, 16, 2, 1, 20000, 512, 512, "bf16", True, 0),
    ("verify_g4_l12", 1, 8, 2, 12, 4096, 512, 512, "f16", False, 0),
    ("verify_g4_l64", 1, 8, 2, 64, 3000, 512, 512, "f16", False, 0),
    ("prefill_causal", 1, 4, 2, 300, 300, 512, 512, "bf16", True, 0),
    ("prefill_window", 1, 4, 2, 333, 333, 512, 512, "bf16", True, 100),
    ("prefill_l_lt_s", 1, 2, 1, 200, 517, 512, 512, "bf16", True, 0),
    ("noncausal_l_gt_s", 1, 2, 2, 90, 40, 512, 512, "bf16", False, 0),
    ("dqk320_dv128", 1, 8, 2, 7, 999, 320, 128, "bf16", True, 0),
    ("dqk128_dv384", 1, 8, 4, 40, 640, 128, 384, "f16", True, 0),
    ("dqk512_dv64", 1, 4, 1, 16, 257, 512, 64, "bf16", False, 0),
    ("d264_ragged", 1, 3, 3, 50, 101, 264, 264, "bf16", True, 17),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_wide_vs_oracle(cuda_lib, case):
    name, B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W = case
    p = I.Problem(B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W, None, 51, name)
    _, _, info = check_problem(cuda_lib, p, force_path=S.PATH_WIDE)
    assert info["path"] == S.PATH_WIDE


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_tc_column_halves_vs_oracle(cuda_lib, case):
    name, B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W = case
    p = I.Problem(B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W, None, 55, name)
    _, _, info = check_problem(cuda_lib, p, force_path=S.PATH_TC)
    assert info["path"] == S.PATH_TC and info["key_block"] == 32


@pytest.mark.parametrize("splits", [1, 3, 0])
def test_tc_column_halves_key_splits(cuda_lib, splits):
    p = I.Problem(1, 8, 2, 40, 6000, 512, 512, "bf16", True, 0, None, 56, "halves_split")
    _, _, info = check_problem(cuda_lib, p, force_path=S.PATH_TC, force_splits=splits)
    assert info["path"] == S.PATH_TC
    if splits:
        assert info["splits"] == splits


def test_tc_column_halves_agree_with_wide(cuda_lib):
    p = I.Problem(1, 4, 2, 200, 700, 512, 512, "bf16", True, 0, None, 57, "halves_agree")
    q, k, v = I.make_qkv(p)
    a = run_gpu(cuda_lib, p, q, k, v, force_path=S.PATH_TC)[0].float()
    b = run_gpu(cuda_lib, p, q, k, v, force_path=S.PATH_WIDE)[0].float()
    assert agree(a, b, "bf16")


@pytest.mark.parametrize("splits", [1, 3, 7, 0])
def test_wide_key_splits(cuda_lib, splits):
    p = I.Problem(1, 16, 2, 2, 5000, 512, 512, "bf16", True, 0, None, 52, "wide_split")
    _, _, info = check_problem(cuda_lib, p, force_splits=splits)
    assert info["path"] == S.PATH_WIDE
    if splits:
        assert info["splits"] == splits


def test_wide_splits_agree(cuda_lib):
    p = I.Problem(1, 16, 1, 1, 8192, 512, 512, "bf16", True, 0, None, 53, "wide_agree")
    q, k, v = I.make_qkv(p)
    a = run_gpu(cuda_lib, p, q, k, v, force_splits=1)[0].float()
    b = run_gpu(cuda_lib, p, q, k, v, force_splits=9)[0].float()
    assert agree(a, b, "bf16")


@pytest.mark.parametrize("path", [S.PATH_WIDE, S.PATH_TC, S.PATH_TC2])
def test_wide_sinks_offset_lse(cuda_lib, path):
    p = I.Problem(1, 4, 2, 40, 700, 512, 512, "bf16", True, 150, None, 54, "wide_ex")
    q, k, v = I.make_qkv(p)
    sinks = [0.25, -2.0, 1.5, 0.0]
    # the pair kernel does not split the keys at head dims above 256
    for fs in ((1,) if path == S.PATH_TC2 else (1, 4)):
        lse = torch.full((1, 4, 40), float("nan"), dtype=torch.float32, device="cuda")
        out = cuda_lib.forward_ex(q.cuda(), k.cuda(), v.cuda(), scale=p.sm_scale, causal=True,
                                  window_size=150, q_offset=500,
                                  sinks=torch.tensor(sinks, device="cuda"), lse=lse,
                                  force_path=path, force_splits=fs)
        cuda_lib.device_status()
        ref, ref_lse = sdpa_oracle(q, k, v, p.sm_scale, True, 150, q_offset=500, sinks=sinks,
                                   return_lse=True)
        err = np.abs(out.float().cpu().numpy() - ref)
        assert err.max() <= TOL_MAX["bf16"] and err.mean() <= TOL_MEAN
        assert np.abs(lse.cpu().numpy() - ref_lse).max() <= 2e-3


@pytest.mark.parametrize("idx", [0, 1, 2])
def test_wide_bench_workloads(cuda_lib, idx):
    """The head-dim-512 bench workloads at full size; the prefill on 256 sampled
    query rows per head."""
    p = I.wide_problems()[idx]
    rows = I.sample_rows(p.L, 256, seed=p.seed) if p.L > 256 else None
    _, _, info = check_problem(cuda_lib, p, rows=rows)
    # decode on the wide path; the prefill's rows fill 256-row pair tiles
    assert info["path"] == (S.PATH_TC2 if p.L > 64 else S.PATH_WIDE)


PAIR_CASES = [
    # name, B, Hq, Hkv, L, S, Dqk, Dv, dtype, causal, window
    ("pair_one_tile", 1, 2, 1, 128, 256, 512, 512, "bf16", True, 0),
    ("pair_ragged_f16", 1, 2, 2, 300, 333, 512, 512, "f16", False, 0),
    ("pair_window", 1, 4, 2, 400, 700, 512, 512, "bf16", True, 150),
    ("pair_window_1", 1, 2, 2, 260, 260, 512, 512, "bf16", True, 1),
    ("pair_dqk320_dv384", 1, 2, 1, 260, 300, 320, 384, "bf16", True, 0),
    ("pair_dqk512_dv264", 1, 2, 2, 256, 190, 512, 264, "f16", False, 0),
    ("pair_many_tiles", 2, 8, 4, 512, 512, 512, 512, "bf16", True, 0),
    ("pair_l_lt_s", 1, 4, 4, 300, 1000, 512, 512, "bf16", True, 0),
]


@pytest.mark.parametrize("case", PAIR_CASES, ids=[c[0] for c in PAIR_CASES])
def test_pair_column_halves_vs_oracle(cuda_lib, case):
    name, B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W = case
    p = I.Problem(B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W, None, 57, name)
    _, _, info = check_problem(cuda_lib, p, force_path=S.PATH_TC2)
    assert info["path"] == S.PATH_TC2 and info["key_block"] == 64 and info["splits"] == 1


@pytest.mark.parametrize("case", PAIR_CASES[:4], ids=[c[0] for c in PAIR_CASES[:4]])
def test_pair_column_halves_agree_with_one_sm(cuda_lib, case):
    name, B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W = case
    p = I.Problem(B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W, None, 58, name)
    q, k, v = I.make_qkv(p)
    a = run_gpu(cuda_lib, p, q, k, v, force_path=S.PATH_TC2)[0].float()
    b = run_gpu(cuda_lib, p, q, k, v, force_path=S.PATH_TC, force_splits=1)[0].float()
    assert agree(a, b, dt)
