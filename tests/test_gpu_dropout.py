"""Dropout parity on the GPU: fa_fwd_dropout / fa_bwd_dropout against the
fp64 oracle's dropout branch.

Two kinds of check:
* the keep mask itself, bit for bit: with Q = 0 every visible key has the
  same probability, so with V = I the forward's O[i, j] is nonzero exactly
  where (query i, key j) is kept, and with dO = I the backward's dV[j, i] is;
* O, LSE, dQ, dK, dV on random inputs within the stated tolerances."""
import math

import numpy as np
import pytest
import torch

import exact_tiled_attention_31_b200 as fa
from oracle import attention as oa
from helpers import check_grad, check_lse, check_o, f64

pytestmark = pytest.mark.gpu


def _rand(B, H, S, D, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float16
    return [torch.randn(B, H, S, D, generator=g).to(dt) for _ in range(4)]


def _mask_inputs(H, dev, dtype=torch.bfloat16):
    S = D = 128
    q = torch.zeros(1, H, S, D, dtype=dtype, device=dev)
    k = torch.randn(1, H, S, D, generator=torch.Generator().manual_seed(1)).to(dtype).to(dev)
    eye = torch.eye(S, dtype=dtype, device=dev).expand(1, H, S, D).contiguous()
    return q, k, eye


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("p,seed,offset", [(0.1, 42, 0), (0.5, (1 << 40) + 3, 77), (0.9, 5, (1 << 33) + 9)])
def test_forward_mask_is_the_oracle_mask(cuda_device, causal, p, seed, offset):
    H = 4
    q, k, eye = _mask_inputs(H, cuda_device)
    o, _ = fa.forward(q, k, eye, causal, 0.1, dropout_p=p, seed=seed, offset=offset)
    fa.check_device_error()
    got = f64(o)[0] != 0
    for h in range(H):
        want = oa.dropout_keep(h, np.arange(128), np.arange(128), p, seed, offset)
        if causal:
            want &= np.tril(np.ones((128, 128), dtype=bool))
        assert np.array_equal(got[h], want), f"head {h}: {np.sum(got[h] != want)} mask bits differ"


@pytest.mark.parametrize("causal", [False, True])
def test_backward_mask_is_the_oracle_mask(cuda_device, causal):
    H, p, seed, offset = 4, 0.3, 1234, 5
    q, k, eye = _mask_inputs(H, cuda_device)
    v = torch.randn(1, H, 128, 128, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16).to(cuda_device)
    o, lse = fa.forward(q, k, v, causal, 0.1, dropout_p=p, seed=seed, offset=offset)
    dq, dk, dv = fa.backward(q, k, v, o, eye, lse, causal, 0.1, dropout_p=p, seed=seed, offset=offset)
    fa.check_device_error()
    got = f64(dv)[0] != 0  # dV[j, i] = P_ij M_ij / (1 - p)
    for h in range(H):
        want = oa.dropout_keep(h, np.arange(128), np.arange(128), p, seed, offset)
        if causal:
            want &= np.tril(np.ones((128, 128), dtype=bool))
        assert np.array_equal(got[h].T, want), f"head {h}: {np.sum(got[h].T != want)} mask bits differ"


@pytest.mark.parametrize("B,H,S,D,dtype,causal,p", [
    (2, 4, 300, 64, "bf16", True, 0.1),
    (1, 3, 517, 128, "fp16", False, 0.3),
    (1, 2, 1024, 128, "bf16", True, 0.5),
    (2, 2, 129, 64, "fp16", False, 0.2),
    # the remaining kernel instances (D x dtype x causal)
    (1, 2, 257, 64, "bf16", False, 0.15),
    (1, 2, 384, 64, "fp16", True, 0.25),
    (1, 2, 200, 128, "fp16", True, 0.4),
])
def test_dropout_forward_backward_match_oracle(cuda_device, B, H, S, D, dtype, causal, p):
    q, k, v, do = _rand(B, H, S, D, dtype, seed=S + D)
    scale, seed, offset = 1.0 / math.sqrt(D), 2024, 11
    d = [x.to(cuda_device) for x in (q, k, v, do)]
    o, lse = fa.forward(d[0], d[1], d[2], causal, scale, dropout_p=p, seed=seed, offset=offset)
    dq, dk, dv = fa.backward(d[0], d[1], d[2], o, d[3], lse, causal, scale, dropout_p=p, seed=seed, offset=offset)
    fa.check_device_error()
    ro, rl = oa.attention_forward_dropout(q, k, v, scale, causal, p, seed, offset)
    check_o(o, ro, f"dropout O {B}x{H}x{S}x{D} {dtype} causal={causal} p={p}")
    check_lse(lse, rl, "dropout LSE")
    # the backward takes the kernel's own O (as a training step does); the
    # oracle's gradients are of the same loss at the oracle's O
    g = oa.attention_backward_dropout(q, k, v, do, scale, causal, p, seed, offset)
    for x, r, name in zip((dq, dk, dv), g, ("dQ", "dK", "dV")):
        check_grad(x, r, f"dropout {name} {B}x{H}x{S}x{D} {dtype} causal={causal} p={p}")


def test_dropout_zero_is_the_plain_path(cuda_device):
    q, k, v, do = (x.to(cuda_device) for x in _rand(1, 2, 333, 128, "bf16", seed=3))
    o0, l0 = fa.forward(q, k, v, True)
    o1, l1 = fa.forward(q, k, v, True, dropout_p=0.0, seed=9, offset=9)
    st = fa.fa_fwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o1.data_ptr(), l1.data_ptr(), 1, 2, 333, 128,
                           1 / math.sqrt(128), 1, 0, 0.0, 9, 9, torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    assert torch.equal(o0, o1) and torch.equal(l0, l1)


def test_dropout_deterministic_backward_is_bitwise_repeatable(cuda_device):
    q, k, v, do = (x.to(cuda_device) for x in _rand(1, 4, 1000, 128, "bf16", seed=4))
    o, lse = fa.forward(q, k, v, True, dropout_p=0.2, seed=1, offset=2)
    runs = [fa.backward(q, k, v, o, do, lse, True, deterministic=True, dropout_p=0.2, seed=1, offset=2)
            for _ in range(3)]
    fa.check_device_error()
    for r in runs[1:]:
        for a, b in zip(runs[0], r):
            assert torch.equal(a, b)


@pytest.mark.parametrize("S,D,dtype,causal", [(1, 64, "bf16", True), (129, 128, "fp16", True),
                                             (300, 64, "bf16", False), (257, 128, "bf16", False)])
def test_dropout_deterministic_on_dirty_workspace_matches_oracle(cuda_device, S, D, dtype, causal):
    """The dropout instances of the deterministic backward on a workspace
    full of 0x7F bytes (3.4e38 as fp32), one tile and several, against the
    oracle's dropout gradients."""
    B, H, p, seed, offset = 1, 3, 0.25, 77, 5
    q, k, v, do = _rand(B, H, S, D, dtype, seed=S * D)
    scale = 1.0 / math.sqrt(D)
    d = [x.to(cuda_device) for x in (q, k, v, do)]
    o, lse = fa.forward(d[0], d[1], d[2], causal, scale, dropout_p=p, seed=seed, offset=offset)
    ws = torch.full((fa.fa_bwd_workspace_size(B, H, S, D),), 0x7F, dtype=torch.uint8, device=cuda_device)
    grads = fa.backward(d[0], d[1], d[2], o, d[3], lse, causal, scale, deterministic=True, workspace=ws,
                        dropout_p=p, seed=seed, offset=offset)
    fa.check_device_error()
    g = oa.attention_backward_dropout(q, k, v, do, scale, causal, p, seed, offset)
    for x, r, name in zip(grads, g, ("dQ", "dK", "dV")):
        check_grad(x, r, f"deterministic dropout {name} S={S} D={D} {dtype} causal={causal}")


def test_dropout_full_size_sampled(cuda_device):
    """B1 H32 S4096 D128 causal bf16, p = 0.1: O and LSE of the last head,
    the gradients of another, against the oracle."""
    q, k, v, do = _rand(1, 32, 4096, 128, "bf16", seed=42)
    scale = 1.0 / math.sqrt(128)
    d = [x.to(cuda_device) for x in (q, k, v, do)]
    o, lse = fa.forward(d[0], d[1], d[2], True, scale, dropout_p=0.1, seed=7, offset=1)
    dq, dk, dv = fa.backward(d[0], d[1], d[2], o, d[3], lse, True, scale, dropout_p=0.1, seed=7, offset=1)
    fa.check_device_error()
    ro, rl = oa.attention_forward_dropout(q, k, v, scale, True, 0.1, 7, 1, heads=[(0, 31)])
    check_o(o[0, [31]], ro, "dropout full size O")
    check_lse(lse[0, [31]], rl, "dropout full size LSE")
    g = oa.attention_backward_dropout(q, k, v, do, scale, True, 0.1, 7, 1, heads=[(0, 17)])
    for x, r, name in zip((dq, dk, dv), g, ("dQ", "dK", "dV")):
        check_grad(x[0, [17]], r, f"dropout full size {name}")
