"""C-ABI library: loads, exports what the header declares, validates on the
host and plans without a GPU (CPU only; no compute call is made)."""
import ctypes
import os
import re

import pytest

import scaled_dot_product_13_b200 as sdpa
from scaled_dot_product_13_b200 import inputs as I

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "sdpa.h")).read()
    return sorted(set(re.findall(r"SDPA_API\s+[\w\s\*]*?\b(sdpa_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return sdpa.load_library()


def test_header_declares_entry_points():
    names = _declared_functions()
    for must in ("sdpa_forward", "sdpa_forward_ws", "sdpa_workspace_bytes", "sdpa_plan",
                 "sdpa_status_string", "sdpa_last_error_message", "sdpa_version"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), f"libsdpa.so does not export {name}"


def test_version_and_status_strings(lib):
    assert lib.sdpa_version() >= 100
    for code, name in sdpa.STATUS.items():
        assert lib.sdpa_status_string(code).decode() == name


def _plan_err(**kw):
    args = dict(B=1, Hq=8, Hkv=2, L=4, S=64, Dqk=128, Dv=128, causal=True, window_size=0,
                dtype="bf16", num_sms=148)
    args.update(kw)
    with pytest.raises(sdpa.SdpaError) as ei:
        sdpa.plan(**args)
    return ei.value


@pytest.mark.parametrize("kw,status,words", [
    (dict(Hq=6, Hkv=4), 1, "multiple of Hkv"),
    (dict(L=65, S=64), 1, "L <= S"),
    (dict(window_size=-1), 1, "window_size"),
    (dict(window_size=8, causal=False), 2, "causal"),
    (dict(Dqk=576, Dv=512), 2, "head dims"),
    (dict(Dqk=512, Dv=520), 2, "[8, 512]"),
    (dict(Dqk=72, Dv=100), 2, "multiples of 8"),
    (dict(B=0), 1, ">= 1"),
    (dict(S=0), 1, ">= 1"),
])
def test_invalid_problems_name_the_constraint(kw, status, words):
    e = _plan_err(**kw)
    assert e.status == status
    assert words in e.message


def test_non_causal_long_query_is_allowed():
    info = sdpa.plan(1, 4, 4, 100, 50, 64, 64, causal=False, num_sms=148)
    assert info["rows"] == 100


def test_forward_rejects_null_pointers_before_any_cuda_call(lib):
    st = lib.sdpa_forward(None, None, None, None, 1, 1, 1, 1, 1, 64, 64, 1.0, 0, 0, 0, None)
    assert st == 1
    assert b"non-NULL" in lib.sdpa_last_error_message()


def test_noalloc_rejects_null_pointers_before_any_cuda_call(lib):
    # same order of checks as sdpa_forward: shape, then pointers, then device
    st = lib.sdpa_forward_noalloc(None, None, None, None, 1, 1, 1, 1, 1, 64, 64, 1.0, 0, 0, 0,
                                  None)
    assert st == 1
    assert b"non-NULL" in lib.sdpa_last_error_message()
    st = lib.sdpa_forward_noalloc(0x1000, 0x2000, 0x3000, 0x4000, 1, 6, 4, 1, 1, 64, 64, 1.0, 0,
                                  0, 0, None)
    assert st == 1
    assert b"multiple of Hkv" in lib.sdpa_last_error_message()


def test_forward_rejects_misaligned_pointers(lib):
    st = lib.sdpa_forward(0x1000, 0x2008, 0x3000, 0x4000, 1, 1, 1, 1, 1, 64, 64, 1.0, 0, 0, 0,
                          None)
    assert st == 1
    assert b"16-byte" in lib.sdpa_last_error_message()


def test_forward_rejects_overlapping_output(lib):
    st = lib.sdpa_forward(0x10000, 0x20000, 0x30000, 0x10000, 1, 1, 1, 4, 4, 64, 64, 1.0, 0, 0,
                          0, None)
    assert st == 1
    assert b"overlap" in lib.sdpa_last_error_message()


def test_plan_decode_splits_keys_across_sms():
    # decode, 64 query heads over 4 KV heads: 16 packed rows per KV head
    info = sdpa.plan(1, 64, 4, 1, 32768, 192, 128, causal=True, num_sms=148)
    assert info["rows"] == 16 and info["row_tiles"] == 1
    assert info["splits"] > 1 and info["launches"] == 2
    assert info["ctas"] <= 148 and info["ctas"] >= 100
    assert info["keys_per_split"] * info["splits"] >= 32768
    assert info["workspace_bytes"] > 0


def test_plan_packs_verify_rows_per_kv_head():
    # verify, GQA 32/8: the 4*L rows of one KV head are packed together
    for L in (1, 2, 4, 8, 12, 16, 24, 32, 48, 64):
        info = sdpa.plan(1, 32, 8, L, 16384, 128, 128, causal=False, dtype="f16", num_sms=148)
        assert info["rows"] == 4 * L
        assert info["row_tiles"] * info["row_tile"] >= 4 * L
        assert info["row_tiles"] * info["row_tile"] < 4 * L + info["row_tile"]


def test_plan_two_split_kv_ctas_per_sm_only_for_the_64_row_layout():
    # 33..64 packed rows (four row warps, no key slices) run two CTAs per SM,
    # so the planner fills twice the SM count; 16- and 32-row layouts one
    # (less at most a seventh, where the split count is rounded down to a
    # whole number of the combine's 32-split rounds: 37 -> 32 per KV head).
    # The router sends 33..64 rows to the tcgen05 kernel, so that layout is
    # forced here.
    for L, per_sm in ((4, 1), (8, 1), (12, 2), (16, 2)):
        info = sdpa.plan(1, 32, 8, L, 32768, 128, 128, causal=False, dtype="f16", num_sms=148,
                         force_path=sdpa.PATH_SPLITKV)
        assert info["path"] == sdpa.PATH_SPLITKV
        assert per_sm * 148 * 6 // 7 <= info["ctas"] <= per_sm * 148, (L, info)
        assert (per_sm - 1) * 148 < info["ctas"], (L, info)
    # routed: up to 32 packed rows on the split-KV kernel, from 33 on tcgen05
    for L, path in ((4, sdpa.PATH_SPLITKV), (8, sdpa.PATH_SPLITKV), (9, sdpa.PATH_TC),
                    (12, sdpa.PATH_TC), (16, sdpa.PATH_TC)):
        info = sdpa.plan(1, 32, 8, L, 32768, 128, 128, causal=False, dtype="f16", num_sms=148)
        assert info["path"] == path, (L, info)
    # head dims whose stages do not fit half the shared memory stay at one per SM
    info = sdpa.plan(1, 32, 8, 16, 32768, 256, 256, causal=False, num_sms=148)
    assert info["ctas"] <= 148


def test_plan_forced_splits_and_single_split_needs_no_workspace():
    info = sdpa.plan(1, 8, 2, 3, 1000, 64, 64, causal=True, num_sms=148, force_splits=1)
    assert info["splits"] == 1 and info["workspace_bytes"] == 0 and info["launches"] == 1
    info = sdpa.plan(1, 8, 2, 3, 1000, 64, 64, causal=True, num_sms=148, force_splits=7)
    assert info["splits"] == 7 and info["launches"] == 2


def test_plan_head_dim_instances():
    assert sdpa.plan(1, 16, 16, 1024, 1024, 72, 72, num_sms=148)["dqk_pad"] == 80
    i = sdpa.plan(1, 64, 4, 1, 256, 192, 128, causal=True, num_sms=148)
    assert (i["dqk_pad"], i["dv_pad"]) == (192, 128)
    assert sdpa.plan(1, 16, 8, 2048, 2048, 256, 256, causal=True, window_size=1024,
                     num_sms=148)["dqk_pad"] == 256


def test_workspace_query_without_device_fails_loudly(lib):
    import torch

    if torch.cuda.is_available():
        pytest.skip("CPU-only check")
    n = lib.sdpa_workspace_bytes(1, 64, 4, 1, 32768, 192, 128, 1, 0, 0)
    assert n == 0
    assert lib.sdpa_last_error_message() != b""


def test_forward_without_device_fails_loudly(lib):
    import torch

    if torch.cuda.is_available():
        pytest.skip("CPU-only check")
    st = lib.sdpa_forward(0x10000, 0x20000, 0x30000, 0x40000, 1, 1, 1, 1, 1, 64, 64, 1.0, 0, 0,
                          0, None)
    assert st == 4
    assert b"CUDA" in lib.sdpa_last_error_message() or b"device" in lib.sdpa_last_error_message()


def test_plan_head_dims_above_256():
    # decode at head dim 512: one 16-row group on the wide path, keys split
    info = sdpa.plan(1, 16, 1, 1, 8192, 512, 512, causal=True, num_sms=148)
    assert info["path"] == sdpa.PATH_WIDE and (info["dqk_pad"], info["dv_pad"]) == (512, 512)
    assert info["row_tile"] == 16 and info["key_block"] == 32 and info["splits"] > 1
    # short verify windows (fewer than 65 packed rows) stay on the wide path
    assert sdpa.plan(1, 8, 2, 12, 4096, 512, 512, num_sms=148)["path"] == sdpa.PATH_WIDE
    # prefill: the pair kernel in two column halves, 64-key blocks, never split
    info = sdpa.plan(1, 8, 8, 4096, 4096, 512, 512, causal=True, num_sms=148)
    assert info["path"] == sdpa.PATH_TC2 and info["row_tile"] == 256 and info["key_block"] == 64
    assert info["ctas"] == 8 * 16 * 2 and info["splits"] == 1 and info["workspace_bytes"] == 0
    # too few pair tiles to give every two SMs one: the one-SM kernel in
    # column halves (two CTAs per row tile)
    info = sdpa.plan(1, 4, 4, 512, 512, 512, 512, causal=True, num_sms=148)
    assert info["path"] == sdpa.PATH_TC and info["row_tile"] == 128 and info["key_block"] == 32
    assert info["ctas"] == 4 * 4 * 2
    # few row tiles: keys split, each split at least 256 keys
    info = sdpa.plan(1, 8, 2, 64, 8192, 512, 512, num_sms=148)
    assert info["path"] == sdpa.PATH_TC and info["splits"] > 1
    assert info["keys_per_split"] >= 256 and info["ctas"] == 2 * 2 * 2 * info["splits"]
    # mixed dims above 256 run on the 512/512 instance
    assert sdpa.plan(1, 4, 4, 64, 64, 320, 128, num_sms=148)["path"] == sdpa.PATH_WIDE
    assert sdpa.plan(1, 4, 4, 128, 128, 128, 384, num_sms=148)["path"] == sdpa.PATH_TC
    # the split-KV, two-tile and looping pair kernels do not take them, and
    # the wide path takes nothing else
    for path in (sdpa.PATH_SPLITKV, sdpa.PATH_TC_DUAL, sdpa.PATH_TC_KSPLIT, sdpa.PATH_TC2_LOOP):
        with pytest.raises(sdpa.SdpaError) as ei:
            sdpa.plan(1, 4, 4, 64, 64, 512, 512, num_sms=148, force_path=path)
        assert ei.value.status == 2 and "wide" in ei.value.message
    for path in (sdpa.PATH_TC, sdpa.PATH_TC2):
        assert sdpa.plan(1, 4, 4, 64, 64, 512, 512, num_sms=148,
                         force_path=path)["path"] == path
    # forced onto the pair kernel it never splits
    with pytest.raises(sdpa.SdpaError) as ei:
        sdpa.plan(1, 1, 1, 256, 8192, 512, 512, num_sms=148, force_path=sdpa.PATH_TC2,
                  force_splits=2)
    assert ei.value.status == 2
    with pytest.raises(sdpa.SdpaError) as ei:
        sdpa.plan(1, 4, 4, 64, 64, 256, 256, num_sms=148, force_path=sdpa.PATH_WIDE)
    assert ei.value.status == 2


def test_plan_two_tile_path_for_small_head_dims():
    # 20 heads x 1500 rows at D=64: 120 CTAs of two 128-row tiles
    info = sdpa.plan(1, 20, 20, 1500, 1500, 64, 64, causal=False, num_sms=148)
    assert info["path"] == sdpa.PATH_TC_DUAL and info["row_tile"] == 256 and info["ctas"] == 120
    # too few 256-row tiles to fill half the SMs: one tile per CTA
    info = sdpa.plan(1, 16, 16, 1024, 1024, 72, 72, causal=False, num_sms=148)
    assert info["path"] == sdpa.PATH_TC
    # head dims 128: the one-tile kernel (P shares the scores' TMEM columns in
    # the two-tile kernel there, and it measured slower)
    info = sdpa.plan(1, 16, 16, 4096, 4096, 128, 128, causal=False, num_sms=148)
    assert info["path"] == sdpa.PATH_TC
    # a window trims the two tiles' key ranges differently: one tile per CTA
    info = sdpa.plan(1, 16, 8, 4096, 4096, 128, 128, causal=True, window_size=1024, num_sms=148)
    assert info["path"] == sdpa.PATH_TC
    # head dims above 128 never take it
    with pytest.raises(sdpa.SdpaError) as ei:
        sdpa.plan(1, 4, 4, 512, 512, 192, 128, num_sms=148, force_path=sdpa.PATH_TC_DUAL)
    assert ei.value.status == 2


def test_plan_looping_pair_path():
    # sliding windows over at least twice as many 256-row tiles as SM pairs:
    # the pair kernel loops over its tiles
    for n in (4096, 8192):
        info = sdpa.plan(1, 16, 8, n, n, 256, 256, causal=True, window_size=1024, num_sms=148)
        assert info["path"] == sdpa.PATH_TC2_LOOP and info["splits"] == 1
        assert info["ctas"] == 8 * (2 * n // 256) and info["launches"] == 1
        assert info["workspace_bytes"] == 0
    # between one and two causal (or windowed) pair tiles per SM pair: twice as
    # many 128-row tiles on the one-SM kernel; non-causal tiles keep the pair
    for window in (1024, 512, 0):
        info = sdpa.plan(1, 16, 8, 2048, 2048, 256, 256, causal=True, window_size=window,
                         num_sms=148)
        assert info["path"] == sdpa.PATH_TC and info["splits"] == 1, (window, info)
        assert info["ctas"] == 8 * (2 * 2048 // 128)
    info = sdpa.plan(1, 16, 8, 2048, 2048, 256, 256, causal=False, num_sms=148)
    assert info["path"] == sdpa.PATH_TC2_LOOP
    info = sdpa.plan(1, 16, 16, 1536, 1536, 192, 128, causal=True, window_size=1024, num_sms=148)
    assert info["path"] == sdpa.PATH_TC
    # long causal tiles keep one pair per tile
    info = sdpa.plan(1, 16, 8, 32768, 32768, 256, 256, causal=True, num_sms=148)
    assert info["path"] == sdpa.PATH_TC2
    # fewer tiles than SM pairs: nothing to loop over (the keys are split instead)
    info = sdpa.plan(1, 4, 2, 2048, 2048, 256, 256, causal=True, window_size=1024, num_sms=148)
    assert info["path"] == sdpa.PATH_TC2 and info["splits"] > 1
    # a window wider than a tile's share of short keys still loops; a long one does not
    info = sdpa.plan(1, 16, 8, 8192, 8192, 256, 256, causal=True, window_size=8000, num_sms=148)
    assert info["path"] == sdpa.PATH_TC2
    # forced: never splits, takes the pair instances (head dims zero filled)
    info = sdpa.plan(1, 4, 4, 512, 512, 64, 64, num_sms=148, force_path=sdpa.PATH_TC2_LOOP)
    assert info["path"] == sdpa.PATH_TC2_LOOP and info["dqk_pad"] == 128 and info["splits"] == 1
    info = sdpa.plan(1, 1, 1, 256, 32768, 256, 256, num_sms=148, force_path=sdpa.PATH_TC2_LOOP)
    assert info["splits"] == 1 and info["ctas"] == 1
    with pytest.raises(sdpa.SdpaError) as ei:
        sdpa.plan(1, 1, 1, 256, 32768, 256, 256, num_sms=148, force_path=sdpa.PATH_TC2_LOOP,
                  force_splits=2)
    assert ei.value.status == 2 and "split" in ei.value.message
    with pytest.raises(sdpa.SdpaError) as ei:
        sdpa.plan(1, 4, 4, 64, 64, 512, 512, num_sms=148, force_path=sdpa.PATH_TC2_LOOP)
    assert ei.value.status == 2


def test_plan_rounds_split_counts_to_whole_combine_rounds():
    # the combine merges 32 splits per round: a count within a seventh above a
    # multiple of 32 is rounded down to it, a larger remainder is kept
    info = sdpa.plan(1, 64, 4, 1, 32768, 192, 128, causal=True, num_sms=148)
    assert info["splits"] == 32 and info["ctas"] == 128, info   # 37 -> 32
    info = sdpa.plan(1, 32, 2, 1, 32768, 128, 128, causal=True, num_sms=148)
    assert info["splits"] == 64, info                            # 74 -> 64
    info = sdpa.plan(1, 48, 3, 1, 32768, 128, 128, causal=True, num_sms=148)
    assert 32 < info["splits"] < 64, info                        # 49 stays above 32
    info = sdpa.plan(1, 64, 8, 1, 32768, 192, 128, causal=True, num_sms=148)
    assert info["splits"] == 18, info                            # below 32: unchanged
    # a pinned split count is kept as given
    info = sdpa.plan(1, 64, 4, 1, 32768, 192, 128, causal=True, num_sms=148, force_splits=37)
    assert info["splits"] == 37, info


def test_plan_balance_rule_bounds():
    # pair tiles = B * Hkv * ceil(g * L / 256); causal 256/256 calls with more
    # than num_sms / 2 and fewer than num_sms of them take the one-SM kernel
    def path(hkv, L, causal=True, window=0, dq=256, dv=256, sms=148):
        return sdpa.plan(1, hkv, hkv, L, L, dq, dv, causal=causal, window_size=window,
                         num_sms=sms)["path"]
    assert path(74, 256) == sdpa.PATH_TC2          # 74 tiles: half the SMs
    assert path(75, 256) == sdpa.PATH_TC           # 75
    assert path(147, 256) == sdpa.PATH_TC          # 147
    assert path(148, 256) == sdpa.PATH_TC2         # 148: two per SM pair
    assert path(75, 256, causal=False) != sdpa.PATH_TC
    assert path(75, 256, window=128) == sdpa.PATH_TC
    assert path(75, 256, dq=192, dv=128) == sdpa.PATH_TC
    # the bounds follow the SM count it plans for
    assert path(75, 256, sms=132) == sdpa.PATH_TC and path(66, 256, sms=132) == sdpa.PATH_TC2
    # head dims that never take the pair kernel are unaffected
    assert path(100, 256, dq=128, dv=128) == sdpa.PATH_TC


def test_plan_routes_every_benchmark_configuration():
    # (path, key splits) the router gives each benchmark configuration on 148
    # SMs, as measured and described with the kernels: a change to the routing
    # rules that moves one of them has to show up here
    S, T, P2, W, D, L7 = (sdpa.PATH_SPLITKV, sdpa.PATH_TC, sdpa.PATH_TC2, sdpa.PATH_WIDE,
                          sdpa.PATH_TC_DUAL, sdpa.PATH_TC2_LOOP)
    want = {"tiny_causal_gqa": (T, 1)}
    for s, k4, k8 in ((256, 1, 1), (1024, 8, 8), (4096, 32, 16), (8192, 32, 16),
                      (16384, 32, 18), (32768, 32, 18)):
        want[f"decode_hkv4_s{s}"] = (S, k4)
        want[f"decode_hkv8_s{s}"] = (S, k8)
    for s, mid in ((16384, 16), (32768, 18)):
        for l in (1, 2, 4, 8):
            want[f"verify_s{s}_l{l}"] = (S, 18)
        for l in (12, 16, 24, 32):
            want[f"verify_s{s}_l{l}"] = (T, mid)
        for l in (48, 64):
            want[f"verify_s{s}_l{l}"] = (T, 9)
    want.update({
        "encoder_h20_l1500_d64": (D, 1), "encoder_h16_l1024_d72": (T, 1),
        "encoder_h16_l4096_d72": (D, 1),
        "window_l2048_w1024_d256": (T, 1), "window_l4096_w1024_d256": (L7, 1),
        "window_l8192_w1024_d256": (L7, 1), "causal_l32768_d256": (P2, 1),
        "wide_decode_d512_s8192": (W, 32), "wide_decode_d512_s32768": (W, 128),
        "wide_prefill_d512_l4096": (P2, 1),
    })
    probs = (I.decode_problems() + I.verify_problems() + I.encoder_problems()
             + I.window_problems() + I.wide_problems() + [I.tiny_problem()])
    assert {p.name for p in probs} == set(want)
    for p in probs:
        info = sdpa.plan(p.B, p.Hq, p.Hkv, p.L, p.S, p.Dqk, p.Dv, p.causal, p.window, p.dtype,
                         num_sms=148)
        assert (info["path"], info["splits"]) == want[p.name], (p.name, info)
