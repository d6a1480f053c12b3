"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs, element by element, within the tolerances stated in
``gpu_util``.  Small shapes span several tiles and ragged tails; the
benchmark shapes run at full size (sampled query rows for the largest)."""
import pytest

from scaled_dot_product_13_b200 import inputs as I
from tests.gpu_util import check_problem

pytestmark = pytest.mark.gpu

SMALL = [
    # name, B, Hq, Hkv, L, S, Dqk, Dv, dtype, causal, window
    ("gqa_causal_ragged", 2, 6, 2, 77, 131, 64, 64, "bf16", True, 0),
    ("mha_noncausal_ragged", 1, 3, 3, 70, 200, 128, 128, "f16", False, 0),
    ("decode_192_128", 1, 16, 1, 1, 333, 192, 128, "bf16", True, 0),
    ("decode_g8", 2, 16, 2, 1, 1000, 192, 128, "bf16", True, 0),
    ("verify_l12", 1, 8, 2, 12, 517, 128, 128, "f16", False, 0),
    ("verify_l48_causal", 1, 8, 2, 48, 700, 128, 128, "f16", True, 0),
    ("d72_ragged", 1, 2, 2, 150, 150, 72, 72, "bf16", False, 0),
    ("d256_window", 1, 4, 2, 300, 300, 256, 256, "bf16", True, 37),
    ("d256_window_lt_s", 1, 4, 2, 100, 400, 256, 256, "bf16", True, 130),
    ("d192_full", 1, 2, 1, 90, 90, 192, 192, "f16", True, 0),
    ("window_1", 1, 2, 1, 33, 33, 64, 64, "bf16", True, 1),
    ("window_ge_s", 1, 2, 2, 65, 65, 64, 64, "bf16", True, 1000),
    ("s_eq_1", 1, 2, 1, 1, 1, 64, 64, "bf16", True, 0),
    ("l_gt_s_noncausal", 1, 2, 1, 90, 17, 64, 64, "f16", False, 0),
    ("odd_dims", 1, 4, 2, 40, 96, 40, 24, "bf16", True, 0),
    ("dqk_lt_dv", 1, 4, 1, 20, 128, 64, 128, "f16", False, 0),
    ("batch3", 3, 4, 4, 33, 65, 128, 128, "bf16", True, 0),
    ("kv_2pow_plus1", 1, 4, 2, 8, 16385, 128, 128, "f16", False, 0),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_small_shapes(cuda_lib, case):
    name, B, Hq, Hkv, L, S, Dqk, Dv, dt, causal, W = case
    p = I.Problem(B, Hq, Hkv, L, S, Dqk, Dv, dt, causal, W, None, 11, name)
    check_problem(cuda_lib, p)


def test_tiny_config(cuda_lib):
    check_problem(cuda_lib, I.tiny_problem())


@pytest.mark.parametrize("p", I.decode_problems(), ids=lambda p: p.name)
def test_decode_configs(cuda_lib, p):
    check_problem(cuda_lib, p)


@pytest.mark.parametrize("p", I.verify_problems(), ids=lambda p: p.name)
def test_verify_configs(cuda_lib, p):
    check_problem(cuda_lib, p)


def test_encoder_1500_d64(cuda_lib):
    check_problem(cuda_lib, I.encoder_problems()[0])


def test_encoder_d72_l1024_full(cuda_lib):
    """pairs * (Dqk + Dv) = 16 * 1024^2 * 144 is below 2^33: compared in full."""
    check_problem(cuda_lib, I.encoder_problems()[1])


def test_encoder_d72_l4096_sampled(cuda_lib):
    p = I.encoder_problems()[2]
    check_problem(cuda_lib, p, rows=I.sample_rows(p.L, 256, p.seed))


@pytest.mark.parametrize("idx", [0, 1, 2], ids=["l2048", "l4096", "l8192"])
def test_window_configs(cuda_lib, idx):
    p = I.window_problems()[idx]
    check_problem(cuda_lib, p, rows=I.sample_rows(p.L, 256, p.seed, window=p.window))


def test_causal_32k_d256_sampled(cuda_lib):
    p = I.window_problems()[3]
    check_problem(cuda_lib, p, rows=I.sample_rows(p.L, 256, p.seed))
