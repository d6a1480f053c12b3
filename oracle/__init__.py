"""fp64 CPU oracle for scaled-dot-product attention (TEST INFRASTRUCTURE).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never loads it and
shares no code with it.

``sdpa_oracle`` wraps the plain C implementation in ``sdpa_oracle.c`` (the
materialised definition O = softmax(scale*Q K^T + mask) V in double
precision; see the header of that file for the formula and the passages of
the pages it follows).  ``bruteforce.sdpa_bruteforce`` is an independent
pure-Python restatement used to pin the C code on tiny inputs.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build_oracle, oracle_lib_path

__all__ = ["sdpa_oracle", "build_oracle", "oracle_lib_path", "load_oracle"]

_LIBS: dict[int, ctypes.CDLL] = {}


def load_oracle(mutant: int = 0) -> ctypes.CDLL:
    """Load (building if needed) the oracle shared library.

    ``mutant`` > 0 loads a build with one deliberately planted mistake; only
    the pin tests use it, to show that the pins would catch such a mistake.
    """
    if mutant in _LIBS:
        return _LIBS[mutant]
    path = oracle_lib_path(mutant)
    if not os.path.exists(path) or os.path.getmtime(path) < os.path.getmtime(
        os.path.join(os.path.dirname(__file__), "sdpa_oracle.c")
    ):
        build_oracle(mutant)
    lib = ctypes.CDLL(path)
    f = lib.oracle_sdpa_f64
    dp = ctypes.POINTER(ctypes.c_double)
    i64 = ctypes.c_int64
    f.argtypes = [dp, dp, dp, dp, dp, i64, i64, i64, i64, i64, i64, i64,
                  ctypes.c_double, ctypes.c_int, i64, i64, i64,
                  ctypes.POINTER(ctypes.c_int64), i64, ctypes.c_int]
    f.restype = ctypes.c_int
    g = lib.oracle_sdpa2_f64
    g.argtypes = f.argtypes + [ctypes.c_int, i64, dp]
    g.restype = ctypes.c_int
    lib.oracle_mutant_id.restype = ctypes.c_int
    _LIBS[mutant] = lib
    return lib


def _as_f64(a) -> np.ndarray:
    try:  # torch tensors (any dtype) -> exact float64 values
        import torch

        if isinstance(a, torch.Tensor):
            return np.ascontiguousarray(a.detach().to("cpu", torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def sdpa_oracle(q, k, v, scale: float, causal: bool = False, window: int = 0,
                rows=None, key_range=None, nthreads: int | None = None,
                return_lse: bool = False, mutant: int = 0, q_offset: int | None = None,
                sinks=None):
    """Materialised fp64 attention.

    q [B,Hq,L,Dqk], k [B,Hkv,S,Dqk], v [B,Hkv,S,Dv] (numpy or torch, any float
    dtype; the values are taken exactly).  ``rows``: optional list of query
    indices; the output then has ``len(rows)`` rows per head.  ``key_range``:
    optional (lo, hi) restricting the keys, as one split of a split-KV pass
    sees them.  ``q_offset``: key position of query row 0 (default S - L).
    ``sinks``: optional [Hq] sink logits (natural-log units).
    Returns O [B,Hq,rows,Dv] float64 (and LSE [B,Hq,rows]).
    """
    qd, kd, vd = _as_f64(q), _as_f64(k), _as_f64(v)
    B, Hq, L, Dqk = qd.shape
    Bk, Hkv, S, Dk2 = kd.shape
    Dv = vd.shape[3]
    if (Bk, Dk2) != (B, Dqk) or vd.shape[:3] != (B, Hkv, S):
        raise ValueError("oracle: inconsistent shapes")
    if rows is None:
        rows_arr = None
        nrows = L
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        nrows = int(rows_arr.size)
    lo, hi = (0, S) if key_range is None else (int(key_range[0]), int(key_range[1]))
    out = np.zeros((B, Hq, nrows, Dv), dtype=np.float64)
    lse = np.zeros((B, Hq, nrows), dtype=np.float64)
    lib = load_oracle(mutant)
    dp = ctypes.POINTER(ctypes.c_double)
    nt = nthreads if nthreads is not None else (os.cpu_count() or 1)
    sk = None if sinks is None else np.ascontiguousarray(_as_f64(sinks).reshape(-1))
    if sk is not None and sk.size != Hq:
        raise ValueError("oracle: sinks must have Hq entries")
    rc = lib.oracle_sdpa2_f64(
        qd.ctypes.data_as(dp), kd.ctypes.data_as(dp), vd.ctypes.data_as(dp),
        out.ctypes.data_as(dp), lse.ctypes.data_as(dp),
        B, Hq, Hkv, L, S, Dqk, Dv, float(scale), int(bool(causal)), int(window),
        lo, hi,
        rows_arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)) if rows_arr is not None else None,
        nrows, int(nt), int(q_offset is not None), int(q_offset or 0),
        sk.ctypes.data_as(dp) if sk is not None else None)
    if rc != 0:
        raise ValueError(f"oracle_sdpa_f64 returned {rc}")
    return (out, lse) if return_lse else out
