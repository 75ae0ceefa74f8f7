"""FP16 range stress on the GPU ("ops-transformer里的FlashAttention", "实战踩坑
坑三" is about FP16 overflow): Q and K drawn N(0,1)*8, so scaled scores reach
about +-64 and products q.k about +-700 before scaling, through the forward
and the backward, dense and packed, against the fp64 oracle on the identical
fp16 inputs."""
import math

import pytest

import exact_tiled_attention_31_b200 as fa
from exact_tiled_attention_31_b200 import inputs
from oracle import attention as oa
from helpers import check_grad, check_lse, check_o, to_dev

pytestmark = pytest.mark.gpu


def test_fp16_stress_dense_s4096_d128_causal(cuda_device):
    """B1 H4 S4096 D128 causal, fp16, Q/K x 8: O, LSE, dQ, dK, dV of two heads."""
    scale = 1 / math.sqrt(128)
    t = inputs.make_dense(1, 4, 4096, 128, "fp16", seed=42, qk_mult=8.0, with_do=True)
    d = to_dev(t, cuda_device)
    o, lse = fa.forward(d["q"], d["k"], d["v"], True, scale)
    dq, dk, dv = fa.backward(d["q"], d["k"], d["v"], o, d["do"], lse, True, scale)
    fa.check_device_error()
    heads = [(0, 0), (0, 3)]
    o_ref, l_ref = oa.attention_forward(t["q"], t["k"], t["v"], scale, True, heads=heads)
    check_lse(lse[0, [0, 3]], l_ref, "fp16 stress LSE")
    check_o(o[0, [0, 3]], o_ref, "fp16 stress O")
    g_ref = oa.attention_backward(t["q"], t["k"], t["v"], t["do"], scale, True, heads=heads)
    for g, r, name in zip((dq, dk, dv), g_ref, ("dQ", "dK", "dV")):
        check_grad(g[0, [0, 3]], r, f"fp16 stress {name}")


def test_fp16_stress_packed_batch(cuda_device):
    """The packed stress batch (32 sequences, lengths uniform in [128, 4096],
    H16 D64 causal, Q/K x 8) in fp16: every sequence of two heads, forward
    and backward."""
    t = inputs.make_varlen(32, 128, 4096, 16, 64, "fp16", seed=42, qk_mult=8.0, with_do=True)
    d = to_dev(t, cuda_device)
    cu = t["cu_seqlens"].to(cuda_device)
    L = max(t["lengths"])
    o, lse = fa.forward_varlen(d["q"], d["k"], d["v"], cu, L, True, 0.125)
    grads = fa.backward_varlen(d["q"], d["k"], d["v"], o, d["do"], lse, cu, L, True, 0.125)
    fa.check_device_error()
    heads = [0, 15]
    o_ref, l_ref = oa.varlen_forward(t["q"], t["k"], t["v"], t["cu_seqlens"], 0.125, True, heads=heads)
    check_lse(lse[heads], l_ref, "fp16 packed LSE")
    check_o(o[heads], o_ref, "fp16 packed O")
    g_ref = oa.varlen_backward(t["q"], t["k"], t["v"], t["do"], t["cu_seqlens"], 0.125, True, heads=heads)
    for g, r, name in zip(grads, g_ref, ("dQ", "dK", "dV")):
        check_grad(g[heads], r, f"fp16 packed {name}")
