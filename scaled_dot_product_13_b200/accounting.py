"""Work accounting for the bench: FLOPs, bytes and pairs of one attention call.

FLOPs count 2*(Dqk+Dv) per unmasked (query, key) pair, exactly (no padding,
no skipped blocks).  KV bytes count the keys visible to at least one query
row of the call, once per KV head.
"""
from __future__ import annotations

from .inputs import Problem


def visible_pairs(p: Problem) -> int:
    """Number of unmasked (query, key) pairs per (batch, query head).

    Counting only, used for FLOP accounting: row i at position
    pos = i + S - L sees keys j in [lo, hi] with hi = pos if causal else S-1 and
    lo = max(0, pos - W + 1) if W else 0.
    """
    total = 0
    off = p.S - p.L
    for i in range(p.L):
        pos = i + off
        hi = pos if p.causal else p.S - 1
        lo = max(0, pos - p.window + 1) if p.window else 0
        total += max(0, hi - lo + 1)
    return total


def visible_key_span(p: Problem) -> int:
    """Keys visible to at least one query row (the union), per (batch, KV head)."""
    off = p.S - p.L
    hi = (p.L - 1 + off) if p.causal else p.S - 1
    lo = max(0, off - p.window + 1) if p.window else 0
    return max(0, hi - lo + 1)


def flops(p: Problem) -> float:
    """2*(Dqk+Dv) FLOPs per unmasked pair, counted exactly."""
    return 2.0 * (p.Dqk + p.Dv) * p.B * p.Hq * visible_pairs(p)


def kv_bytes(p: Problem) -> float:
    """Bytes of K and V the call must read: the visible key span of every KV head."""
    return float(p.B * p.Hkv * visible_key_span(p) * (p.Dqk + p.Dv) * 2)


def io_bytes(p: Problem) -> float:
    """Q read + O written, bytes."""
    return float(p.B * p.Hq * p.L * (p.Dqk + p.Dv) * 2)


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)
