"""GPU invariants the pages fix, checked on the CUDA path itself: the result
does not depend on the split count or the route; GQA equals explicitly
repeated KV heads; window >= S equals plain causal; a decode row equals the
last row of the causal prefill.  Plus the device watchdog and error paths."""
import numpy as np
import pytest
import torch

from scaled_dot_product_13_b200 import inputs as I
from tests.gpu_util import agree, TOL_MAX, TOL_MEAN, check_problem, run_gpu

pytestmark = pytest.mark.gpu



def _out(sdpa, p, q, k, v, **kw):
    return run_gpu(sdpa, p, q, k, v, **kw)[0].float()


@pytest.mark.parametrize("splits", [1, 2, 7, 0, 10_000])
def test_split_count_invariance(cuda_lib, splits):
    p = I.Problem(1, 16, 2, 3, 3000, 192, 128, "bf16", True, 0, None, 5, "splits")
    check_problem(cuda_lib, p, force_splits=splits)


def test_splits_agree_with_each_other(cuda_lib):
    p = I.Problem(1, 8, 2, 10, 2500, 128, 128, "f16", False, 0, None, 6)
    q, k, v = I.make_qkv(p)
    outs = [_out(cuda_lib, p, q, k, v, force_splits=s) for s in (1, 2, 7, 39)]
    for o in outs[1:]:
        assert agree(o, outs[0], "f16")


def test_gqa_equals_repeated_kv(cuda_lib):
    p = I.Problem(1, 8, 2, 40, 300, 128, 128, "bf16", True, 0, None, 7)
    q, k, v = I.make_qkv(p)
    a = _out(cuda_lib, p, q, k, v)
    pr = p.with_(Hkv=8)
    b = _out(cuda_lib, pr, q, k.repeat_interleave(4, 1).contiguous(),
             v.repeat_interleave(4, 1).contiguous())
    assert agree(a, b, "bf16")


def test_window_ge_s_equals_causal(cuda_lib):
    p = I.Problem(1, 4, 2, 200, 200, 64, 64, "bf16", True, 0, None, 8)
    q, k, v = I.make_qkv(p)
    a = _out(cuda_lib, p, q, k, v)
    b = _out(cuda_lib, p.with_(window=200), q, k, v)
    c = _out(cuda_lib, p.with_(window=5000), q, k, v)
    assert torch.equal(a, b) and torch.equal(a, c)


def test_decode_equals_last_prefill_row(cuda_lib):
    p = I.Problem(1, 8, 2, 96, 96, 128, 128, "f16", True, 0, None, 9)
    q, k, v = I.make_qkv(p)
    full = _out(cuda_lib, p, q, k, v)
    last = _out(cuda_lib, p.with_(L=1), q[:, :, -1:].contiguous(), k, v)
    assert agree(full[:, :, -1], last[:, :, 0], "f16")


def test_repeated_calls_are_deterministic(cuda_lib):
    p = I.decode_problems()[3]
    q, k, v = I.make_qkv(p)
    a = _out(cuda_lib, p, q, k, v)
    b = _out(cuda_lib, p, q, k, v)
    assert torch.equal(a, b)


def test_default_stream_allocating_entry_point(cuda_lib):
    # sdpa_forward takes its split workspace stream-ordered from the pool
    p = I.decode_problems()[5]
    q, k, v = (t.cuda() for t in I.make_qkv(p))
    out = cuda_lib.forward(q, k, v, scale=p.sm_scale, causal=True)
    cuda_lib.device_status()
    ref, _ = run_gpu(cuda_lib, p, q.cpu(), k.cpu(), v.cpu())
    assert torch.equal(out, ref)


def test_watchdog_expires_cleanly(cuda_lib):
    cuda_lib.device_status(clear=True)
    assert cuda_lib.watchdog_selftest(50_000_000) == 0
    with pytest.raises(cuda_lib.SdpaError) as ei:
        cuda_lib.device_status(clear=True)
    assert ei.value.status == 5
    cuda_lib.device_status(clear=True)  # cleared: healthy again
    # the context is still usable
    check_problem(cuda_lib, I.tiny_problem())


def test_errors_raise_before_launch(cuda_lib):
    q = torch.zeros(1, 4, 8, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 3, 8, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cuda_lib.SdpaError) as ei:
        cuda_lib.forward(q, k, k)
    assert ei.value.status == 1
    k = torch.zeros(1, 4, 4, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cuda_lib.SdpaError) as ei:
        cuda_lib.forward(q, k, k, causal=True)
    assert "L <= S" in ei.value.message
    big = torch.zeros(1, 4, 8, 576, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cuda_lib.SdpaError) as ei:
        cuda_lib.forward(big, big, big)
    assert ei.value.status == 2
    ws = torch.zeros(4, dtype=torch.float32, device="cuda")
    p = I.decode_problems()[5]
    q, k, v = (t.cuda() for t in I.make_qkv(p))
    with pytest.raises(cuda_lib.SdpaError) as ei:
        cuda_lib.forward_ws(q, k, v, ws, scale=p.sm_scale, causal=True)
    assert ei.value.status == 3
