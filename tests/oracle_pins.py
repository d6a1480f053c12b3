"""The checks that pin the fp64 oracle to something other than itself.

Each ``pin_*`` function runs one family of checks against the oracle build
``mutant`` (0 = the real oracle) and returns a list of failure messages
(empty = pass).  ``tests/test_oracle.py`` requires every pin to pass on the
real oracle and at least one pin to fail on every planted-mistake build.

Definition pinned: O = softmax(scale * Q K^T + mask) V with grouped-query
heads, causal masking aligned to the end of the keys and a sliding window of
the last W keys including the query's own (mlx PR #3552; mlx issue #3826).
"""
from __future__ import annotations

import math

import numpy as np
import torch

from oracle import sdpa_oracle
from oracle.bruteforce import sdpa_bruteforce


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _qkv(B, Hq, Hkv, L, S, Dqk, Dv, seed):
    return (_rand((B, Hq, L, Dqk), seed), _rand((B, Hkv, S, Dqk), seed + 1),
            _rand((B, Hkv, S, Dv), seed + 2))


TINY_CASES = [
    # B, Hq, Hkv, L, S, Dqk, Dv, causal, window
    (1, 2, 1, 5, 9, 8, 8, True, 0),
    (1, 2, 2, 7, 7, 16, 8, False, 0),
    (2, 2, 1, 6, 11, 12, 20, True, 4),
    (1, 4, 2, 9, 9, 8, 8, True, 1),
    (1, 3, 1, 1, 13, 24, 16, True, 0),
    (1, 2, 1, 13, 33, 8, 4, True, 7),
    (1, 1, 1, 4, 1, 8, 8, False, 0),
    (1, 2, 2, 3, 17, 8, 8, False, 0),
]


def pin_bruteforce(mutant=0):
    """Oracle vs the pure-Python brute force on tiny inputs (rel 1e-12)."""
    fails = []
    for n, (B, Hq, Hkv, L, S, Dqk, Dv, causal, W) in enumerate(TINY_CASES):
        q, k, v = _qkv(B, Hq, Hkv, L, S, Dqk, Dv, 100 + n)
        scale = Dqk ** -0.5
        ref = np.asarray(sdpa_bruteforce(q.tolist(), k.tolist(), v.tolist(), scale, causal, W))
        got = sdpa_oracle(q, k, v, scale, causal, W, mutant=mutant)
        err = np.max(np.abs(got - ref) / (1e-300 + np.maximum(1.0, np.abs(ref))))
        if not err <= 1e-12:
            fails.append(f"bruteforce case {n}: rel err {err}")
    return fails


def pin_closed_forms(mutant=0):
    """Closed forms the definition fixes exactly."""
    fails = []
    B, Hq, Hkv, L, S, D = 1, 4, 2, 6, 10, 8
    q, k, v = _qkv(B, Hq, Hkv, L, S, D, D, 7)
    for causal, W in ((False, 0), (True, 0), (True, 3)):
        # constant V rows -> O equals that row
        vc = np.broadcast_to(np.arange(D, dtype=np.float64) - 2.5, v.shape).copy()
        o = sdpa_oracle(q, k, vc, 0.3, causal, W, mutant=mutant)
        if not np.allclose(o, vc[:, :1, :1, :].repeat(Hq, 1).repeat(L, 2), atol=1e-13):
            fails.append(f"constant V (causal={causal}, W={W})")
        # identical keys -> mean of V over the visible keys of each row
        kc = np.broadcast_to(k[:, :, :1, :], k.shape).copy()
        o = sdpa_oracle(q, kc, v, 0.3, causal, W, mutant=mutant)
        for hq in range(Hq):
            hk = hq // (Hq // Hkv)
            for i in range(L):
                pos = i + S - L
                hi = pos + 1 if causal else S
                lo = max(0, pos - W + 1) if W else 0
                want = v[0, hk, lo:hi].mean(axis=0)
                if not np.allclose(o[0, hq, i], want, atol=1e-13):
                    fails.append(f"identical keys hq={hq} i={i} causal={causal} W={W}")
                    break
        # q = 0 -> the same uniform average
        o0 = sdpa_oracle(np.zeros_like(q), k, v, 0.3, causal, W, mutant=mutant)
        if not np.allclose(o0, o, atol=1e-13):
            fails.append(f"q=0 uniform average (causal={causal}, W={W})")
    # W = 1 -> each row returns V at its own position
    o = sdpa_oracle(q, k, v, 0.3, True, 1, mutant=mutant)
    for hq in range(Hq):
        hk = hq // (Hq // Hkv)
        for i in range(L):
            if not np.allclose(o[0, hq, i], v[0, hk, i + S - L], atol=1e-13):
                fails.append(f"W=1 hq={hq} i={i}")
                break
    # S = 1 -> O = V[0]
    o = sdpa_oracle(q, k[:, :, :1], v[:, :, :1], 0.3, False, 0, mutant=mutant)
    if not np.allclose(o, v[:, :, :1].repeat(Hq // Hkv, 1).repeat(L, 2), atol=1e-13):
        fails.append("S=1")
    # one key with a huge score margin -> that key's V row
    qh = np.zeros((1, 1, 1, D)); qh[..., 0] = 1.0
    kh = np.zeros((1, 1, S, D)); kh[0, 0, 3, 0] = 1.0
    o = sdpa_oracle(qh, kh, v[:, :1], 800.0, False, 0, mutant=mutant)
    if not np.allclose(o[0, 0, 0], v[0, 0, 3], atol=1e-12):
        fails.append("huge margin key")
    # weights: with V = identity (Dv = S), O[i] is the weight vector; it must
    # sum to 1 and be the softmax of the visible scores
    S2 = 9
    q2, k2, _ = _qkv(1, 2, 1, 4, S2, 8, 8, 11)
    eye = np.eye(S2)[None, None]
    wts = sdpa_oracle(q2, k2, eye, 0.5, True, 0, mutant=mutant)
    if not np.allclose(wts.sum(-1), 1.0, atol=1e-14):
        fails.append("weights do not sum to 1")
    for hq in range(2):
        for i in range(4):
            pos = i + S2 - 4
            s = 0.5 * (k2[0, 0, :pos + 1] @ q2[0, hq, i])
            want = np.exp(s - s.max()); want /= want.sum()
            if not np.allclose(wts[0, hq, i, :pos + 1], want, atol=1e-14) or \
                    np.any(wts[0, hq, i, pos + 1:] != 0):
                fails.append(f"weights hq={hq} i={i}")
    return fails


def pin_invariants(mutant=0):
    """Invariants the pages fix (window >= S is causal; decode equals the last
    prefill row; GQA equals repeated KV heads; key splits merge by LSE)."""
    fails = []
    B, Hq, Hkv, L, S, Dqk, Dv = 1, 6, 2, 12, 12, 16, 24
    q, k, v = _qkv(B, Hq, Hkv, L, S, Dqk, Dv, 21)
    sc = Dqk ** -0.5
    causal = sdpa_oracle(q, k, v, sc, True, 0, mutant=mutant)
    for W in (S, S + 5, 4 * S):
        if not np.allclose(sdpa_oracle(q, k, v, sc, True, W, mutant=mutant), causal, atol=1e-14):
            fails.append(f"window {W} >= S differs from causal")
    # an L=1 query at position S-1 equals the last row of the causal prefill
    last = sdpa_oracle(q[:, :, -1:], k, v, sc, True, 0, mutant=mutant)
    if not np.allclose(last[:, :, 0], causal[:, :, -1], atol=1e-14):
        fails.append("decode row != last prefill row")
    # a windowed decode row equals the last windowed prefill row
    lw = sdpa_oracle(q[:, :, -1:], k, v, sc, True, 5, mutant=mutant)
    fw = sdpa_oracle(q, k, v, sc, True, 5, mutant=mutant)
    if not np.allclose(lw[:, :, 0], fw[:, :, -1], atol=1e-14):
        fails.append("windowed decode row != last windowed prefill row")
    # GQA equals explicitly repeated KV heads (each KV head serves g
    # consecutive query heads)
    g = Hq // Hkv
    kr, vr = np.repeat(k, g, axis=1), np.repeat(v, g, axis=1)
    for c, W in ((False, 0), (True, 0), (True, 4)):
        a = sdpa_oracle(q, k, v, sc, c, W, mutant=mutant)
        b = sdpa_oracle(q, kr, vr, sc, c, W, mutant=mutant)
        if not np.allclose(a, b, atol=1e-14):
            fails.append(f"GQA != repeated KV (causal={c}, W={W})")
    # splitting the keys and merging by log-sum-exp gives the full result
    for c, W in ((False, 0), (True, 0), (True, 5)):
        full, lse_full = sdpa_oracle(q, k, v, sc, c, W, return_lse=True, mutant=mutant)
        cuts = [0, 3, 4, 9, S]
        parts = [sdpa_oracle(q, k, v, sc, c, W, key_range=(a, b), return_lse=True, mutant=mutant)
                 for a, b in zip(cuts[:-1], cuts[1:])]
        lses = np.stack([p[1] for p in parts])
        mx = lses.max(axis=0)
        wts = np.exp(lses - mx)
        lse = mx + np.log(wts.sum(axis=0))
        merged = sum(np.exp(p[1] - lse)[..., None] * p[0] for p in parts)
        if not (np.allclose(merged, full, atol=1e-13) and np.allclose(lse, lse_full, atol=1e-13)):
            fails.append(f"LSE merge of key splits != full (causal={c}, W={W})")
    return fails


def pin_torch_library(mutant=0):
    """Special case that reduces to a library routine: torch's fp64 CPU
    scaled_dot_product_attention given an explicit bottom-right boolean mask
    and explicitly repeated KV heads."""
    fails = []
    cases = [(1, 4, 2, 16, 40, 32, 16, True, 0), (2, 2, 1, 33, 33, 24, 24, True, 9),
             (1, 3, 3, 20, 50, 16, 16, False, 0), (1, 4, 1, 1, 64, 64, 32, True, 0)]
    for n, (B, Hq, Hkv, L, S, Dqk, Dv, causal, W) in enumerate(cases):
        q, k, v = _qkv(B, Hq, Hkv, L, S, Dqk, Dv, 300 + n)
        sc = Dqk ** -0.5
        i = torch.arange(L)[:, None] + (S - L)
        j = torch.arange(S)[None, :]
        mask = torch.ones(L, S, dtype=torch.bool)
        if causal:
            mask &= j <= i
        if W:
            mask &= (i - j) < W
        g = Hq // Hkv
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q), torch.from_numpy(np.repeat(k, g, 1)),
            torch.from_numpy(np.repeat(v, g, 1)), attn_mask=mask, scale=sc).numpy()
        got = sdpa_oracle(q, k, v, sc, causal, W, mutant=mutant)
        err = np.max(np.abs(got - ref))
        if not err <= 1e-12:
            fails.append(f"torch sdpa case {n}: max abs err {err}")
    return fails


def pin_lse(mutant=0):
    """The LSE output equals log(sum_j exp(s_j)) over the visible keys,
    computed directly (small scores, no max subtraction)."""
    fails = []
    q, k, v = _qkv(1, 2, 1, 5, 8, 8, 8, 41)
    sc = 8 ** -0.5
    _, lse = sdpa_oracle(q, k, v, sc, True, 3, return_lse=True, mutant=mutant)
    for hq in range(2):
        for i in range(5):
            pos = i + 3
            js = [j for j in range(8) if j <= pos and pos - j < 3]
            want = math.log(math.fsum(math.exp(sc * float(q[0, hq, i] @ k[0, 0, j])) for j in js))
            if abs(lse[0, hq, i] - want) > 1e-12:
                fails.append(f"lse hq={hq} i={i}")
    return fails


OFFSET_SINK_CASES = [
    # B, Hq, Hkv, L, S, D, causal, W, q_offset, sinks
    (1, 2, 1, 5, 9, 8, True, 0, 2, None),
    (1, 2, 1, 4, 12, 8, True, 3, 6, None),
    (1, 2, 2, 6, 6, 8, True, 0, None, [0.7, -1.5]),
    (1, 4, 2, 3, 10, 8, True, 4, 5, [1.0, 2.0, -3.0, 0.0]),
    (2, 2, 1, 7, 7, 12, False, 0, None, [0.3, 0.9]),
    (1, 2, 1, 9, 4, 8, True, 0, 0, [0.2, 0.1]),  # more queries than keys, offset 0
]


def pin_offset_and_sinks(mutant=0):
    """Query offset (chunked prefill, rotating cache) and sinks against the
    brute force, the chunked-prefill and rotating-cache invariants, and a
    library cross-check of sinks."""
    fails = []
    for n, (B, Hq, Hkv, L, S, D, causal, W, off, sk) in enumerate(OFFSET_SINK_CASES):
        q, k, v = _qkv(B, Hq, Hkv, L, S, D, D, 500 + n)
        sc = D ** -0.5
        ref = np.asarray(sdpa_bruteforce(q.tolist(), k.tolist(), v.tolist(), sc, causal, W,
                                         q_offset=off, sinks=sk))
        got = sdpa_oracle(q, k, v, sc, causal, W, q_offset=off, sinks=sk, mutant=mutant)
        if not np.max(np.abs(got - ref)) <= 1e-12:
            fails.append(f"offset/sink brute force case {n}")
    # q_offset = S - L is the default alignment
    q, k, v = _qkv(1, 2, 1, 5, 11, 8, 8, 531)
    for c, W in ((True, 0), (True, 4)):
        a = sdpa_oracle(q, k, v, 0.4, c, W, mutant=mutant)
        b = sdpa_oracle(q, k, v, 0.4, c, W, q_offset=6, mutant=mutant)
        if not np.array_equal(a, b):
            fails.append("q_offset = S - L differs from the default")
    # chunked prefill: queries [c0, c1) over keys [0, c1) with offset c0 are
    # rows [c0, c1) of the full causal (and windowed) prefill
    N = 24
    q, k, v = _qkv(1, 2, 1, N, N, 8, 8, 532)
    for W in (0, 5):
        full = sdpa_oracle(q, k, v, 0.4, True, W, mutant=mutant)
        for c0, c1 in ((0, 8), (8, 16), (16, 24), (5, 13)):
            part = sdpa_oracle(q[:, :, c0:c1], k[:, :, :c1], v[:, :, :c1], 0.4, True, W,
                               q_offset=c0, mutant=mutant)
            if not np.allclose(part, full[:, :, c0:c1], atol=1e-14):
                fails.append(f"chunked prefill rows [{c0},{c1}) W={W}")
    # rotating window cache: only the last W + chunk - 1 keys are held; with
    # positions relative to the first held key the result is unchanged
    W, c0, c1 = 6, 14, 20
    first = c0 - W + 1
    full = sdpa_oracle(q, k, v, 0.4, True, W, mutant=mutant)
    part = sdpa_oracle(q[:, :, c0:c1], k[:, :, first:c1], v[:, :, first:c1], 0.4, True, W,
                       q_offset=c0 - first, mutant=mutant)
    if not np.allclose(part, full[:, :, c0:c1], atol=1e-14):
        fails.append("rotating window cache")
    # sinks: -inf is no sink; weights plus the sink's weight sum to 1
    q, k, v = _qkv(1, 2, 1, 4, 9, 8, 8, 533)
    if not np.array_equal(sdpa_oracle(q, k, v, 0.5, True, 0, sinks=[-np.inf, -np.inf], mutant=mutant),
                          sdpa_oracle(q, k, v, 0.5, True, 0, mutant=mutant)):
        fails.append("sink -inf differs from no sink")
    eye = np.eye(9)[None, None]
    wts, lse = sdpa_oracle(q, k, eye, 0.5, True, 0, sinks=[0.4, 1.7], return_lse=True,
                           mutant=mutant)
    w_sink = np.exp(np.array([0.4, 1.7])[None, :, None] - lse)
    if not np.allclose(wts.sum(-1) + w_sink, 1.0, atol=1e-14):
        fails.append("weights + sink weight != 1")
    # library: the sink is one more key with a zero row whose score is set by
    # an additive float mask; torch's fp64 SDPA then gives the same O
    q, k, v = _qkv(1, 4, 2, 6, 10, 8, 8, 534)
    sinks = np.array([0.3, -0.8, 1.2, 2.0])
    g = 2
    i = np.arange(6)[:, None] + 4
    j = np.arange(10)[None, :]
    bias = np.where(j <= i, 0.0, -np.inf)
    kk = np.concatenate([np.repeat(k, g, 1), np.zeros((1, 4, 1, 8))], axis=2)
    vv = np.concatenate([np.repeat(v, g, 1), np.zeros((1, 4, 1, 8))], axis=2)
    mask = np.concatenate([np.broadcast_to(bias, (1, 4, 6, 10)),
                           np.broadcast_to(sinks[None, :, None, None], (1, 4, 6, 1))], axis=3)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(kk), torch.from_numpy(vv),
        attn_mask=torch.from_numpy(np.ascontiguousarray(mask)), scale=0.35).numpy()
    got = sdpa_oracle(q, k, v, 0.35, True, 0, sinks=sinks, mutant=mutant)
    if not np.max(np.abs(got - ref)) <= 1e-12:
        fails.append("sinks vs torch extra-key construction")
    return fails


ALL_PINS = [pin_bruteforce, pin_closed_forms, pin_invariants, pin_torch_library, pin_lse,
            pin_offset_and_sinks]
