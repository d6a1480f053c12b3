"""sdpa_forward_noalloc against sdpa_forward (GPU).

The no-allocation entry point serves callers that cannot call cudaMalloc or
cudaMallocAsync: split partials go to the library's fixed per-device scratch
array instead of a workspace the call or the caller allocates.  Its output
must match the allocating entry point within the GPU tolerance, on two calls
in a row that follow a call on other inputs of the same shape (so the scratch
holds stale partials that differ from the right ones).  This file is collected last so that a stop at the first failure
has already run every other test; it also passes on its own in a fresh
process.
"""
import pytest
import torch

from scaled_dot_product_13_b200 import inputs as I
from tests.gpu_util import TOL_MAX

pytestmark = pytest.mark.gpu

CASES = [
    # split over the keys (partials in scratch), bf16 decode, 192/128 dims
    I.Problem(1, 64, 8, 1, 32768, 192, 128, "bf16", True, 0, 192 ** -0.5, 1, "decode_hkv8_s32768"),
    # fp16 verify window with packed GQA rows, split
    I.Problem(1, 32, 8, 16, 16384, 128, 128, "f16", False, 0, 128 ** -0.5, 2, "verify_s16384_l16"),
    # causal prefill with a window; the plan may not split (scratch unused)
    I.Problem(1, 4, 2, 300, 300, 64, 64, "bf16", True, 37, None, 3, "window_prefill"),
]


@pytest.mark.parametrize("p", CASES, ids=lambda p: p.name)
def test_noalloc_matches_allocating_entry_point(cuda_lib, p):
    q, k, v = (t.cuda() for t in I.make_qkv(p))
    ref = cuda_lib.forward(q, k, v, scale=p.sm_scale, causal=p.causal, window_size=p.window)
    cuda_lib.device_status()
    # leave partials of other inputs in the shared scratch first, so that an
    # element the attention pass failed to write would show up as a mismatch
    other = torch.empty_like(ref)
    cuda_lib.forward_noalloc(-q, k.flip(2), v * 0.5, scale=p.sm_scale, causal=p.causal,
                             window_size=p.window, out=other)
    cuda_lib.device_status()
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        cuda_lib.forward_noalloc(q, k, v, scale=p.sm_scale, causal=p.causal,
                                 window_size=p.window, out=out)
        cuda_lib.device_status()
        err = (out.float() - ref.float()).abs().max().item()
        assert err <= TOL_MAX[p.dtype], f"{p.name}: max abs diff {err}"


def test_noalloc_rejects_problems_beyond_the_scratch(cuda_lib):
    # one full 128-row tile whose 64K keys are split across every SM: the
    # fp32 partials (splits x 128 rows x 256 columns) exceed 16 MiB
    p = I.Problem(1, 2, 1, 64, 65536, 256, 256, "bf16", False, 0, None, 4, "big")
    need = cuda_lib.workspace_bytes(p.B, p.Hq, p.Hkv, p.L, p.S, p.Dqk, p.Dv, p.causal,
                                    p.window, p.dtype)
    if need <= (16 << 20):
        pytest.skip(f"plan on this device needs only {need} bytes of scratch")
    q = torch.zeros(p.B, p.Hq, p.L, p.Dqk, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(p.B, p.Hkv, p.S, p.Dqk, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cuda_lib.SdpaError) as ei:
        cuda_lib.forward_noalloc(q, k, k, causal=False)
    assert ei.value.status == 3 and "maximum" in ei.value.message
