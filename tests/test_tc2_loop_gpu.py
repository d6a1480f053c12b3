"""GPU parity of the looping form of the two-CTA kernel (SDPA_PATH_TC2_LOOP:
at most one CTA pair per two SMs, each walking several 256-row tiles with the
next tile's Q and first scores issued under the current tile's end) against
the oracle.  The looping form does the same arithmetic in the same order as
one pair per tile, so its output must equal that path's bit for bit."""
import numpy as np
import pytest
import torch

import scaled_dot_product_13_b200 as S
from oracle import sdpa_oracle
from scaled_dot_product_13_b200 import inputs as I
from tests.gpu_util import TOL_MAX, TOL_MEAN, check_problem, run_gpu
from tests.test_tc2_gpu import CASES

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_loop_vs_oracle(cuda_lib, case):
    name, B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W = case
    p = I.Problem(B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W, None, 51, name)
    _, _, info = check_problem(cuda_lib, p, force_path=S.PATH_TC2_LOOP)
    assert info["path"] == S.PATH_TC2_LOOP and info["splits"] == 1


# More 256-row tiles than SM pairs, so every pair walks two to seven tiles:
# both Q buffers are reused, block and tile counters run across tiles, and
# tiles of different lengths (causal, window edges, ragged ends) follow each
# other in one pair.
WALK = [
    # name, B, Hq, Hkv, L, S, Dqk, Dv, dtype, causal, window
    ("walk_window_d256", 4, 16, 8, 2048, 2048, 256, 256, "bf16", True, 1024),
    ("walk_window_ragged_f16", 3, 8, 4, 1900, 2100, 256, 256, "f16", True, 333),
    ("walk_causal_d256", 2, 16, 16, 1024, 1024, 256, 256, "bf16", True, 0),
    ("walk_noncausal_gqa", 3, 32, 8, 512, 640, 256, 256, "bf16", False, 0),
    ("walk_d192_128_window", 2, 16, 4, 1500, 1500, 192, 128, "bf16", True, 512),
    ("walk_d128_window", 2, 32, 8, 1200, 1300, 128, 128, "f16", True, 200),
    ("walk_window_1", 2, 8, 8, 2304, 2304, 256, 256, "bf16", True, 1),
]


@pytest.mark.parametrize("case", WALK, ids=[c[0] for c in WALK])
def test_loop_walks_many_tiles(cuda_lib, case):
    name, B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W = case
    p = I.Problem(B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W, None, 52, name)
    q, k, v = I.make_qkv(p)
    a, info = run_gpu(cuda_lib, p, q, k, v, force_path=S.PATH_TC2_LOOP)
    assert info["path"] == S.PATH_TC2_LOOP and info["ctas"] > 74
    # every row of tile boundaries, the ragged end and a spread of others
    rows = sorted(set(r for r in (0, 1, 127, 128, 255, 256, 511, 512, L // 3, L // 2, L - 257,
                                  L - 256, L - 129, L - 128, L - 2, L - 1) if 0 <= r < L))
    ref = sdpa_oracle(q, k, v, p.sm_scale, causal, W, rows=rows)
    got = a.float().cpu().numpy()[:, :, rows]
    err = np.abs(got - ref)
    assert err.max() <= TOL_MAX[dt] and err.mean() <= TOL_MEAN, (err.max(), err.mean())
    b, info2 = run_gpu(cuda_lib, p, q, k, v, force_path=S.PATH_TC2, force_splits=1)
    assert info2["path"] == S.PATH_TC2 and info2["splits"] == 1
    assert torch.equal(a, b), "looping form differs from one pair per tile"


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_loop_equals_one_pair_per_tile(cuda_lib, case):
    name, B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W = case
    p = I.Problem(B, Hq, Hkv, L, Sk, Dqk, Dv, dt, causal, W, None, 53, name)
    q, k, v = I.make_qkv(p)
    a = run_gpu(cuda_lib, p, q, k, v, force_path=S.PATH_TC2_LOOP)[0]
    # unsplit, as the looping form (few tiles would otherwise split the keys)
    b = run_gpu(cuda_lib, p, q, k, v, force_path=S.PATH_TC2, force_splits=1)[0]
    assert torch.equal(a, b)


def test_loop_sinks_offset_lse(cuda_lib):
    # a chunk of 900 queries at positions 450.. over 1400 keys, 4 heads on 2
    p = I.Problem(1, 4, 2, 900, 1400, 256, 256, "bf16", True, 200, None, 54, "loop_ex")
    q, k, v = I.make_qkv(p)
    sinks = [0.5, -1.0, 2.0, 0.0]
    lse = torch.full((1, 4, 900), float("nan"), dtype=torch.float32, device="cuda")
    out = cuda_lib.forward_ex(q.cuda(), k.cuda(), v.cuda(), scale=p.sm_scale, causal=True,
                              window_size=200, q_offset=450,
                              sinks=torch.tensor(sinks, device="cuda"), lse=lse,
                              force_path=S.PATH_TC2_LOOP)
    cuda_lib.device_status()
    ref, ref_lse = sdpa_oracle(q, k, v, p.sm_scale, True, 200, q_offset=450, sinks=sinks,
                               return_lse=True)
    err = np.abs(out.float().cpu().numpy() - ref)
    assert err.max() <= TOL_MAX["bf16"] and err.mean() <= TOL_MEAN
    assert np.abs(lse.cpu().numpy() - ref_lse).max() <= 2e-3


@pytest.mark.parametrize("scale", [-0.05, 0.0, 0.3])
def test_loop_unusual_scales(cuda_lib, scale):
    p = I.Problem(2, 8, 4, 700, 700, 256, 256, "bf16", True, 100, scale, 55, "loop_scales")
    check_problem(cuda_lib, p, force_path=S.PATH_TC2_LOOP)


def test_loop_rejects_splits(cuda_lib):
    p = I.Problem(1, 2, 1, 256, 2048, 256, 256, "bf16", True, 0, None, 56, "loop_split")
    q, k, v = I.make_qkv(p)
    with pytest.raises(S.SdpaError) as ei:
        run_gpu(cuda_lib, p, q, k, v, force_path=S.PATH_TC2_LOOP, force_splits=3)
    assert ei.value.status == 2
