"""Host-side error paths, exercised by fault injection on the host (GPU).

The library reads two test-only variables when it loads:
SDPA_TEST_FAIL_ALLOC makes the stream-ordered workspace allocation of the
allocating entry point fail, and SDPA_TEST_SMEM_LIMIT makes the pre-launch
resource check (the counterpart of the dispatch-time threadgroup-size check
of mlx PR #4185, "Kernel support") compare against a smaller shared-memory
limit.  Each case runs in a child process with the variable set.  The call
must fail with the documented status and a message, enqueue nothing (its
output buffer keeps its sentinel), and leave the context usable.  No GPU
fault, trap or hang is involved."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys, torch
sys.path.insert(0, {root!r})
import scaled_dot_product_13_b200 as sdpa
from scaled_dot_product_13_b200 import inputs as I
sdpa.load_library()
p = I.Problem(1, 64, 8, 1, 4096, 192, 128, "bf16", True, 0, 192 ** -0.5, 1, "decode")
q, k, v = (t.cuda() for t in I.make_qkv(p))
out = torch.full((1, 64, 1, 128), 7.0, dtype=torch.bfloat16, device="cuda")
try:
    sdpa.{call}
    print("STATUS 0")
except sdpa.SdpaError as e:
    print("STATUS", e.status)
    print("MESSAGE", e.message)
torch.cuda.synchronize()
print("UNTOUCHED", bool((out == 7.0).all().item()))
# the context still computes: the caller-owned workspace path needs neither
# the allocation nor (without the limit) the refused check
ws = torch.empty(max(sdpa.workspace_bytes(1, 64, 8, 1, 4096, 192, 128, True), 4) // 4,
                 dtype=torch.float32, device="cuda")
try:
    sdpa.forward_ws(q, k, v, ws, scale=p.sm_scale, causal=True, out=out)
    torch.cuda.synchronize()
    print("AFTER", bool(torch.isfinite(out.float()).all().item()))
except sdpa.SdpaError as e:
    print("AFTER_STATUS", e.status)
"""


def _run(env_extra, call):
    env = dict(os.environ)
    env.update(env_extra)
    code = CHILD.format(root=ROOT, call=call)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    return dict(line.split(" ", 1) for line in r.stdout.strip().splitlines())


def test_injected_allocation_failure(cuda_lib):
    res = _run({"SDPA_TEST_FAIL_ALLOC": "1"},
               "forward(q, k, v, scale=p.sm_scale, causal=True, out=out)")
    assert res["STATUS"] == "4"
    assert "cudaMallocAsync" in res["MESSAGE"] and "injected" in res["MESSAGE"]
    assert res["UNTOUCHED"] == "True"
    assert res["AFTER"] == "True"


def test_injected_resource_refusal(cuda_lib):
    res = _run({"SDPA_TEST_SMEM_LIMIT": "1024"},
               "forward(q, k, v, scale=p.sm_scale, causal=True, out=out)")
    assert res["STATUS"] == "3"
    assert "shared memory" in res["MESSAGE"]
    assert res["UNTOUCHED"] == "True"
    # the limit stays in force for the workspace path too: refused again
    assert res.get("AFTER_STATUS") == "3"
