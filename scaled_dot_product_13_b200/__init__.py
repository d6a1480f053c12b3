"""Python binding of libsdpa (argument marshalling only).

Every computation happens in the CUDA kernels of ``libsdpa.so``; this module
only checks tensor metadata, passes device pointers, sizes and the current
CUDA stream to the C ABI declared in ``include/sdpa.h``, and turns a status
code into an exception.  There is no CPU or PyTorch fallback: if the library
or a CUDA device is missing, calls raise.

    import scaled_dot_product_13_b200 as sdpa
    out = sdpa.forward(q, k, v, scale=None, causal=True, window_size=0)

q [B, Hq, L, Dqk], k [B, Hkv, S, Dqk], v [B, Hkv, S, Dv], contiguous CUDA
tensors of one dtype (bfloat16 or float16).  Query head hq reads KV head
hq // (Hq // Hkv); query i sits at key position i + S - L.
"""
from __future__ import annotations

import ctypes
import os

__all__ = ["forward", "forward_ws", "forward_noalloc", "forward_ex", "Options", "workspace_bytes", "plan", "device_status",
           "set_wait_limit_ns", "watchdog_selftest", "exp2_selftest", "time_next_main_kernel", "time_next_call", "load_library", "library_path",
           "SdpaError", "PATH_AUTO", "PATH_SPLITKV", "PATH_TC", "PATH_TC2", "PATH_WIDE", "PATH_TC_DUAL", "PATH_TC_KSPLIT",
           "PATH_TC2_LOOP", "STATUS"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB: ctypes.CDLL | None = None

PATH_AUTO, PATH_SPLITKV, PATH_TC, PATH_TC2, PATH_WIDE, PATH_TC_DUAL, PATH_TC_KSPLIT, PATH_TC2_LOOP = \
    0, 1, 2, 3, 4, 5, 6, 7
STATUS = {0: "SDPA_OK", 1: "SDPA_ERR_INVALID_ARG", 2: "SDPA_ERR_UNSUPPORTED",
          3: "SDPA_ERR_RESOURCES", 4: "SDPA_ERR_CUDA", 5: "SDPA_ERR_TIMEOUT"}


class SdpaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status
        self.message = message


class Options(ctypes.Structure):
    """Mirror of sdpa_options."""
    _fields_ = [("has_q_offset", ctypes.c_int), ("q_offset", ctypes.c_int),
                ("sinks", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("force_path", ctypes.c_int), ("force_splits", ctypes.c_int)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int), ("splits", ctypes.c_int), ("rows", ctypes.c_int),
                ("row_tile", ctypes.c_int), ("row_tiles", ctypes.c_int),
                ("key_block", ctypes.c_int), ("keys_per_split", ctypes.c_int),
                ("ctas", ctypes.c_int), ("launches", ctypes.c_int), ("dqk_pad", ctypes.c_int),
                ("dv_pad", ctypes.c_int), ("workspace_bytes", ctypes.c_size_t)]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


def library_path() -> str:
    return os.environ.get("SDPA_LIBRARY", os.path.join(_HERE, "libsdpa.so"))


def load_library() -> ctypes.CDLL:
    """Load libsdpa.so (raises if it was not built)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"libsdpa.so not found at {path}; build it with "
                           "`python -m scaled_dot_product_13_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    common = [vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, i, i]
    lib.sdpa_forward.argtypes = common + [vp]
    lib.sdpa_forward_ws.argtypes = common + [vp, sz, vp]
    lib.sdpa_forward_noalloc.argtypes = common + [vp]
    lib.sdpa_forward_ex.argtypes = common + [ctypes.POINTER(Options), vp, sz, vp]
    lib.sdpa_forward_planned.argtypes = common + [i, i, vp, sz, vp]
    lib.sdpa_workspace_bytes.argtypes = [i] * 10
    lib.sdpa_workspace_bytes.restype = sz
    lib.sdpa_plan.argtypes = [i] * 13 + [ctypes.POINTER(PlanInfo)]
    lib.sdpa_device_status.argtypes = [i]
    lib.sdpa_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.sdpa_set_wait_limit_ns.restype = None
    lib.sdpa_watchdog_selftest.argtypes = [ctypes.c_uint64, ctypes.POINTER(ctypes.c_int)]
    lib.sdpa_exp2_selftest.argtypes = [ctypes.c_float, ctypes.c_float, i, vp, vp]
    lib.sdpa_time_next_main_kernel.argtypes = [vp, vp]
    lib.sdpa_time_next_main_kernel.restype = None
    lib.sdpa_time_next_call.argtypes = [vp, vp, vp]
    lib.sdpa_time_next_call.restype = None
    lib.sdpa_status_string.restype = ctypes.c_char_p
    lib.sdpa_status_string.argtypes = [i]
    lib.sdpa_last_error_message.restype = ctypes.c_char_p
    for fn in ("sdpa_forward", "sdpa_forward_ws", "sdpa_forward_noalloc", "sdpa_forward_ex",
               "sdpa_forward_planned", "sdpa_plan",
               "sdpa_device_status", "sdpa_watchdog_selftest", "sdpa_exp2_selftest"):
        getattr(lib, fn).restype = ctypes.c_int
    _LIB = lib
    return lib


def _check(status: int) -> None:
    if status != 0:
        msg = load_library().sdpa_last_error_message().decode(errors="replace")
        raise SdpaError(status, msg)


def _dtype_code(t) -> int:
    import torch

    if t.dtype == torch.bfloat16:
        return 0
    if t.dtype == torch.float16:
        return 1
    raise SdpaError(2, f"dtype {t.dtype} is not supported (bfloat16 or float16)")


def _shapes(q, k, v):
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise SdpaError(1, "q, k, v must be 4-D [B, H, N, D]")
    B, Hq, L, Dqk = q.shape
    Bk, Hkv, S, Dk = k.shape
    Bv, Hv, Sv, Dv = v.shape
    if (Bk, Dk) != (B, Dqk) or (Bv, Hv, Sv) != (B, Hkv, S):
        raise SdpaError(1, f"inconsistent shapes q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda:
            raise SdpaError(1, f"{name} must be a CUDA tensor")
        if not t.is_contiguous():
            raise SdpaError(1, f"{name} must be contiguous")
        if t.dtype != q.dtype:
            raise SdpaError(1, "q, k, v must share one dtype")
    return int(B), int(Hq), int(Hkv), int(L), int(S), int(Dqk), int(Dv)


def _stream(stream):
    import torch

    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _out_like(q, L, Dv, out):
    import torch

    B, Hq = q.shape[0], q.shape[1]
    if out is None:
        return torch.empty((B, Hq, L, Dv), dtype=q.dtype, device=q.device)
    if tuple(out.shape) != (B, Hq, L, Dv) or out.dtype != q.dtype or not out.is_contiguous():
        raise SdpaError(1, "out must be a contiguous [B, Hq, L, Dv] tensor of q's dtype")
    return out


def forward(q, k, v, scale: float | None = None, causal: bool = False, window_size: int = 0,
            out=None, stream=None):
    """Fused attention forward; returns out [B, Hq, L, Dv] (same dtype as q)."""
    lib = load_library()
    B, Hq, Hkv, L, S, Dqk, Dv = _shapes(q, k, v)
    sc = float(Dqk ** -0.5 if scale is None else scale)
    out = _out_like(q, L, Dv, out)
    _check(lib.sdpa_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, Hq,
                            Hkv, L, S, Dqk, Dv, sc, int(bool(causal)), int(window_size),
                            _dtype_code(q), _stream(stream)))
    return out


def forward_noalloc(q, k, v, scale: float | None = None, causal: bool = False,
                    window_size: int = 0, out=None, stream=None):
    """As ``forward``, through sdpa_forward_noalloc: no device allocation in
    the library; split partials go to the library's fixed 16 MiB per-device
    scratch array.  ``out`` should be preallocated by callers that cannot
    allocate (when None, this wrapper allocates it with torch).  Calls that
    overlap on the GPU share that array and race; keep them on one stream."""
    lib = load_library()
    B, Hq, Hkv, L, S, Dqk, Dv = _shapes(q, k, v)
    sc = float(Dqk ** -0.5 if scale is None else scale)
    out = _out_like(q, L, Dv, out)
    _check(lib.sdpa_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B,
                                    Hq, Hkv, L, S, Dqk, Dv, sc, int(bool(causal)),
                                    int(window_size), _dtype_code(q), _stream(stream)))
    return out


def forward_ex(q, k, v, scale: float | None = None, causal: bool = False, window_size: int = 0,
               q_offset: int | None = None, sinks=None, lse=None, out=None, stream=None,
               workspace=None, force_path: int = 0, force_splits: int = 0):
    """sdpa_forward_ex: ``q_offset`` = key position of query row 0 (default
    S - L); ``sinks`` = optional float32 CUDA tensor [Hq] of sink logits;
    ``lse`` = optional float32 CUDA tensor [B, Hq, L] that receives each row's
    log-sum-exp.  ``workspace``: as ``forward_ws`` (None = pool allocation)."""
    import torch

    lib = load_library()
    B, Hq, Hkv, L, S, Dqk, Dv = _shapes(q, k, v)
    sc = float(Dqk ** -0.5 if scale is None else scale)
    out = _out_like(q, L, Dv, out)
    opt = Options()
    if q_offset is not None:
        opt.has_q_offset, opt.q_offset = 1, int(q_offset)
    for name, t, shape in (("sinks", sinks, (Hq,)), ("lse", lse, (B, Hq, L))):
        if t is None:
            continue
        if not (t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()
                and tuple(t.shape) == shape):
            raise SdpaError(1, f"{name} must be a contiguous float32 CUDA tensor of shape {shape}")
    opt.sinks = sinks.data_ptr() if sinks is not None else None
    opt.lse = lse.data_ptr() if lse is not None else None
    opt.force_path, opt.force_splits = int(force_path), int(force_splits)
    ws_ptr = 0 if workspace is None else workspace.data_ptr()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.sdpa_forward_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, Hq,
                               Hkv, L, S, Dqk, Dv, sc, int(bool(causal)), int(window_size),
                               _dtype_code(q), ctypes.byref(opt), ws_ptr, ws_bytes,
                               _stream(stream)))
    return out


def forward_ws(q, k, v, workspace, scale: float | None = None, causal: bool = False,
               window_size: int = 0, out=None, stream=None, force_path: int = 0,
               force_splits: int = 0):
    """As ``forward`` with a caller-owned workspace tensor (any dtype, on the
    device, at least ``workspace_bytes`` bytes; may be None when that is 0).
    ``force_path`` / ``force_splits`` pin the router (0 = its choice)."""
    lib = load_library()
    B, Hq, Hkv, L, S, Dqk, Dv = _shapes(q, k, v)
    sc = float(Dqk ** -0.5 if scale is None else scale)
    out = _out_like(q, L, Dv, out)
    ws_ptr = 0 if workspace is None else workspace.data_ptr()
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.sdpa_forward_planned(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                    B, Hq, Hkv, L, S, Dqk, Dv, sc, int(bool(causal)),
                                    int(window_size), _dtype_code(q), int(force_path),
                                    int(force_splits), ws_ptr, ws_bytes, _stream(stream)))
    return out


def workspace_bytes(B, Hq, Hkv, L, S, Dqk, Dv, causal=False, window_size=0, dtype="bf16",
                    force_path: int = 0, force_splits: int = 0, num_sms: int | None = None) -> int:
    """Workspace a call needs (router's plan, or the pinned one)."""
    return plan(B, Hq, Hkv, L, S, Dqk, Dv, causal, window_size, dtype, num_sms=num_sms,
                force_path=force_path, force_splits=force_splits)["workspace_bytes"]


def plan(B, Hq, Hkv, L, S, Dqk, Dv, causal=False, window_size=0, dtype="bf16",
         num_sms: int | None = None, force_path: int = 0, force_splits: int = 0) -> dict:
    """The router's decision for one problem (host only)."""
    lib = load_library()
    if num_sms is None:
        num_sms = _num_sms()
    info = PlanInfo()
    dt = 0 if dtype in ("bf16", "bfloat16") else 1
    _check(lib.sdpa_plan(B, Hq, Hkv, L, S, Dqk, Dv, int(bool(causal)), int(window_size), dt,
                         int(num_sms), int(force_path), int(force_splits), ctypes.byref(info)))
    return info.as_dict()


def _num_sms() -> int:
    try:
        import torch

        if torch.cuda.is_available():
            return torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    except Exception:  # pragma: no cover
        pass
    return 148


def device_status(clear: bool = True) -> None:
    """Synchronise and raise SdpaError(SDPA_ERR_TIMEOUT) if a kernel's bounded
    wait expired since the last clear."""
    _check(load_library().sdpa_device_status(int(bool(clear))))


def time_next_main_kernel(start_event, stop_event) -> None:
    """Arm the profiling hook: the next call on this thread records the two
    torch.cuda.Event objects around its main attention kernel.  The events
    must already hold a CUDA handle (record them once beforehand)."""
    if not start_event.cuda_event or not stop_event.cuda_event:
        raise SdpaError(1, "events have no CUDA handle yet; record them once first")
    load_library().sdpa_time_next_main_kernel(ctypes.c_void_p(start_event.cuda_event),
                                              ctypes.c_void_p(stop_event.cuda_event))


def time_next_call(start_event, stop_event, call_event) -> None:
    """As ``time_next_main_kernel``, plus ``call_event`` recorded after the
    call's last launch (the combine, when the keys are split).  Any of the
    three may be None (not recorded)."""
    handles = []
    for e in (start_event, stop_event, call_event):
        if e is not None and not e.cuda_event:
            raise SdpaError(1, "events have no CUDA handle yet; record them once first")
        handles.append(ctypes.c_void_p(e.cuda_event if e is not None else None))
    load_library().sdpa_time_next_call(*handles)


def exp2_selftest(lo: float, hi: float, n: int, device="cuda"):
    """(poly, ref): the kernels' FMA-pipe exp2 and exp2f on n points over
    [lo, hi], as fp32 CUDA tensors."""
    import torch

    poly = torch.empty(n, dtype=torch.float32, device=device)
    ref = torch.empty(n, dtype=torch.float32, device=device)
    _check(load_library().sdpa_exp2_selftest(ctypes.c_float(lo), ctypes.c_float(hi), int(n),
                                             ctypes.c_void_p(poly.data_ptr()),
                                             ctypes.c_void_p(ref.data_ptr())))
    torch.cuda.synchronize()
    return poly, ref


def set_wait_limit_ns(ns: int) -> None:
    load_library().sdpa_set_wait_limit_ns(int(ns))


def watchdog_selftest(limit_ns: int = 100_000_000) -> int:
    """Run the watchdog self-test kernel; returns 0 when its wait expired."""
    res = ctypes.c_int(-1)
    _check(load_library().sdpa_watchdog_selftest(int(limit_ns), ctypes.byref(res)))
    return res.value
