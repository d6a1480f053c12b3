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


ALL_PINS = [pin_bruteforce, pin_closed_forms, pin_invariants, pin_torch_library, pin_lse]
