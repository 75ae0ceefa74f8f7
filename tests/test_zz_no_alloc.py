"""The allocation-free backward (fa_bwd_noalloc) against the regular one.

Callers that cannot allocate device memory (allocator hooks, fixed memory
budgets, latency-critical loops) use fa_bwd_noalloc, which keeps its scratch
in the library's fixed device array instead of a caller workspace.  It must
give the same gradients as fa_bwd, call after call, even though every call
reuses the previous call's scratch contents.

This file is named so that pytest collects it last; it also passes when run
on its own in a fresh process.
"""
import math

import pytest
import torch

import exact_tiled_attention_31_b200 as fa
from exact_tiled_attention_31_b200 import inputs
from helpers import check_grad, to_dev


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """Checked on the host before anything is launched (no GPU needed)."""
    A = 1 << 20  # 16-byte aligned fake address, never dereferenced
    B, H, S, D = 1, 32, 4096, 128
    assert fa.fa_bwd_workspace_size(B, H, S, D) > fa.api.NOALLOC_SCRATCH_BYTES
    st = fa.fa_bwd_noalloc(*([A] * 9), B, H, S, D, 0.088, 1, fa.api.FA_BF16, 0, None)
    assert st == fa.api.FA_ERR_UNSUPPORTED


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,S,D,causal,dtype,det", [
    (1, 8, 1024, 128, True, "bf16", False),
    (2, 4, 777, 64, False, "fp16", False),
    (1, 4, 640, 128, True, "bf16", True),
])
def test_noalloc_matches_regular_backward_twice(cuda_device, B, H, S, D, causal, dtype, det):
    assert fa.fa_bwd_workspace_size(B, H, S, D) <= fa.api.NOALLOC_SCRATCH_BYTES
    scale = 1 / math.sqrt(D)
    t = to_dev(inputs.make_dense(B, H, S, D, dtype, seed=S + D, with_do=True), cuda_device)
    o, lse = fa.forward(t["q"], t["k"], t["v"], causal, scale)
    ref = fa.backward(t["q"], t["k"], t["v"], o, t["do"], lse, causal, scale, deterministic=det)
    for _ in range(2):
        dq, dk, dv = (torch.full_like(t["q"], float("nan")) for _ in range(3))
        fa.backward_noalloc(t["q"], t["k"], t["v"], o, t["do"], lse, dq, dk, dv, causal, scale, deterministic=det)
        fa.check_device_error()
        for got, want, name in zip((dq, dk, dv), ref, ("dQ", "dK", "dV")):
            check_grad(got, want, f"{name} noalloc vs regular")
            if det:
                assert torch.equal(got, want), f"{name}: deterministic results differ"
