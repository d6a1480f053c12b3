"""Pure-Python brute force used to pin the C oracle (TEST INFRASTRUCTURE).

A second, deliberately different restatement of the same definition: it
loops over (b, hq, i, j) with ``math.exp`` on the raw scores (no max
subtraction, so it is only valid for small scores), sums with ``math.fsum``
and builds the visibility test from positions rather than from the C code's
helper.  It is slow (pure Python) and meant for B*H <= 4, L, S <= ~40.

Definition followed: O = softmax(scale * Q K^T + mask) V, GQA head
hk = floor(hq / (Hq/Hkv)) (mlx issue #3826, routing analysis), causal with
queries aligned to the end of the keys (mlx PR #3552, qL_off = kL - qL) and a
window of the last W key positions including the query's own (mlx PR #3552,
Summary).
"""
from __future__ import annotations

import math


def sdpa_bruteforce(q, k, v, scale, causal=False, window=0, q_offset=None, sinks=None):
    """q, k, v: nested lists or arrays [B][H][N][D] of Python floats.
    ``q_offset``: key position of query 0 (default S - L).  ``sinks``: per
    query head logit that joins the normalisation without a value row."""
    B = len(q)
    Hq = len(q[0])
    L = len(q[0][0])
    Hkv = len(k[0])
    S = len(k[0][0])
    Dv = len(v[0][0][0])
    g = Hq // Hkv
    out = []
    for b in range(B):
        ob = []
        for hq in range(Hq):
            hk = hq // g
            oh = []
            for i in range(L):
                pos = (S - L if q_offset is None else q_offset) + i
                keys = [j for j in range(S)
                        if (not causal or j <= pos) and (window == 0 or j > pos - window)]
                ws = []
                for j in keys:
                    s = math.fsum(float(a) * float(c) for a, c in zip(q[b][hq][i], k[b][hk][j]))
                    ws.append(math.exp(scale * s))
                den = math.fsum(ws + ([math.exp(float(sinks[hq]))] if sinks is not None else []))
                row = [math.fsum(w * float(v[b][hk][j][d]) for w, j in zip(ws, keys)) / den
                       for d in range(Dv)]
                oh.append(row)
            ob.append(oh)
        out.append(ob)
    return out
