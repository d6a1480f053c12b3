"""Host-side helpers of bench.py (CPU): the verify sweep's monotonicity and
cliff checks, and the traffic line lookup."""
import bench


def _pts(S, times):
    Ls = (1, 2, 4, 8, 12, 16, 24, 32, 48, 64)
    return [{"name": f"verify_s{S}_l{L}", "us": t} for L, t in zip(Ls, times)]


def test_verify_checks_pass_a_smooth_sweep():
    pts = _pts(32768, [32.1, 33.2, 33.7, 36.2, 42.2, 42.3, 47.9, 48.3, 59.2, 61.1])
    c = bench.verify_checks(pts)["s32768"]
    assert c["monotone"] and c["no_cliff"]
    assert c["worst_step"]["from_L"] == 32 and c["worst_step"]["to_L"] == 48


def test_verify_checks_flag_the_pages_cliff():
    # a 2.3x jump for 1.5x the rows between L=8 and L=12
    pts = _pts(16384, [10, 10, 10, 10, 23, 24, 26, 28, 33, 36])
    c = bench.verify_checks(pts)["s16384"]
    assert c["monotone"] and not c["no_cliff"]
    assert c["worst_step"] == {"from_L": 8, "to_L": 12, "ratio": 2.3}


def test_verify_checks_flag_a_drop():
    # L=32 more than 3 % faster than L=24
    pts = _pts(16384, [22, 22, 23, 26, 30, 30, 34, 32, 41, 43])
    c = bench.verify_checks(pts)["s16384"]
    assert not c["monotone"] and c["no_cliff"]


def test_verify_checks_keep_each_sequence_length_apart():
    pts = _pts(16384, [22] * 10) + _pts(32768, [32] * 10)
    c = bench.verify_checks(pts)
    assert set(c) == {"s16384", "s32768"}


def test_traffic_line_lookup():
    # a recorded launch gives bytes while its kernel source is unchanged, else
    # None (the bench then reports traffic = null); an unknown launch is None
    got = bench.ncu_traffic("splitkv.cuh", "decode_hkv8_s32768")
    assert got is None or (isinstance(got, int) and got > 167_772_160)
    assert bench.ncu_traffic("splitkv.cuh", "no_such_launch") is None
