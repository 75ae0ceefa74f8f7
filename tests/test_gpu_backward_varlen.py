"""Backward parity on the GPU for packed variable-length batches ([H, T, D]
with cu_seqlens): dQ, dK, dV from fa_bwd_varlen against the fp64 oracle,
which runs the textbook gradients one sequence at a time."""
import numpy as np
import pytest
import torch

import exact_tiled_attention_31_b200 as fa
from exact_tiled_attention_31_b200 import inputs
from oracle import attention as oa
from helpers import check_grad, to_dev

pytestmark = pytest.mark.gpu


def _run(t, causal, scale, dev, deterministic=False):
    d = to_dev(t, dev)
    cu = t["cu_seqlens"].to(dev)
    max_len = max(t["lengths"])
    o, lse = fa.forward_varlen(d["q"], d["k"], d["v"], cu, max_len, causal, scale)
    grads = fa.backward_varlen(d["q"], d["k"], d["v"], o, d["do"], lse, cu, max_len, causal, scale,
                               deterministic=deterministic)
    fa.check_device_error()
    return grads


def _check(t, causal, scale, grads, heads, what):
    ref = oa.varlen_backward(t["q"], t["k"], t["v"], t["do"], t["cu_seqlens"], scale, causal, heads=heads)
    for g, r, name in zip(grads, ref, ("dQ", "dK", "dV")):
        check_grad(g[heads], r, f"{name} {what}")


def _pack(lengths, H, D, dtype, seed):
    """A packed batch with the given lengths (q, k, v, dO ~ N(0,1), rounded)."""
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T = int(cu[-1])
    g = torch.Generator().manual_seed(seed)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float16
    out = {k: torch.randn(H, T, D, generator=g).to(dt) for k in ("q", "k", "v", "do")}
    out.update(lengths=list(lengths), cu_seqlens=torch.tensor(cu), total=T)
    return out


def test_bwd_varlen_packed_batch(cuda_device):
    """32 sequences, lengths uniform in [128, 4096], H=16 D=64 causal, Q and K
    drawn N(0,1)*8 (scores up to +-64): every sequence of two heads."""
    t = inputs.make_varlen(32, 128, 4096, 16, 64, "bf16", seed=42, qk_mult=8.0, with_do=True)
    grads = _run(t, True, 0.125, cuda_device)
    _check(t, True, 0.125, grads, [0, 15], "packed batch")


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_varlen_small_mixed(cuda_device, causal):
    """Short, ragged and single-token sequences in one pack, D=128, fp16."""
    t = _pack([1, 5, 128, 129, 300, 17, 256, 2], 4, 128, "fp16", seed=3)
    grads = _run(t, causal, 0.09, cuda_device)
    _check(t, causal, 0.09, grads, [0, 1, 2, 3], f"mixed causal={causal}")


def test_bwd_varlen_d64_bf16_noncausal(cuda_device):
    t = _pack([200, 64, 513, 1, 130], 2, 64, "bf16", seed=11)
    grads = _run(t, False, 0.125, cuda_device)
    _check(t, False, 0.125, grads, [0, 1], "D=64 bf16 non-causal")


def test_bwd_varlen_one_sequence_equals_dense(cuda_device):
    """A pack holding one sequence is the dense problem with B = 1: dK and dV
    bit for bit, dQ bit for bit under deterministic mode."""
    S, H, D = 700, 3, 128
    t = _pack([S], H, D, "bf16", seed=21)
    d = to_dev(t, cuda_device)
    cu = t["cu_seqlens"].to(cuda_device)
    o_v, lse_v = fa.forward_varlen(d["q"], d["k"], d["v"], cu, S, True, 0.088)
    gv = fa.backward_varlen(d["q"], d["k"], d["v"], o_v, d["do"], lse_v, cu, S, True, 0.088, deterministic=True)
    dense = {k: d[k].unsqueeze(0) for k in ("q", "k", "v", "do")}
    o_d, lse_d = fa.forward(dense["q"], dense["k"], dense["v"], True, 0.088)
    gd = fa.backward(dense["q"], dense["k"], dense["v"], o_d, dense["do"], lse_d, True, 0.088, deterministic=True)
    fa.check_device_error()
    assert torch.equal(o_v, o_d[0]) and torch.equal(lse_v, lse_d[0])
    for a, b, name in zip(gv, gd, ("dQ", "dK", "dV")):
        assert torch.equal(a, b[0]), name


def test_bwd_varlen_deterministic_is_bitwise_repeatable(cuda_device):
    t = _pack([300, 1, 777, 128, 64], 4, 128, "bf16", seed=5)
    runs = [_run(t, True, 0.088, cuda_device, deterministic=True) for _ in range(3)]
    for r in runs[1:]:
        for a, b in zip(runs[0], r):
            assert torch.equal(a, b)
    nd = _run(t, True, 0.088, cuda_device, deterministic=False)
    for a, b, name in zip(runs[0], nd, ("dQ", "dK", "dV")):
        check_grad(b, a, f"{name} atomic vs ordered")
    _check(t, True, 0.088, runs[0], [0, 3], "deterministic")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_varlen_deterministic_on_dirty_workspace(cuda_device, D, causal):
    """Deterministic mode of a packed batch on a workspace full of 0x7F bytes
    (3.4e38 as fp32): one-token, sub-tile, one-tile-plus-one and several-tile
    sequences, so some query tiles have a single key tile (the second chain's
    accumulator gets nothing there) and the packed rows of neighbouring
    sequences share 32-row boxes; against the oracle, every sequence of every
    head."""
    lengths, H = [1, 130, 257, 64, 400], 3
    t = _pack(lengths, H, D, "bf16", seed=11 + D + int(causal))
    d = to_dev(t, cuda_device)
    cu = t["cu_seqlens"].to(cuda_device)
    L, scale = max(lengths), 1.0 / np.sqrt(D)
    o, lse = fa.forward_varlen(d["q"], d["k"], d["v"], cu, L, causal, scale)
    ws = torch.full((fa.fa_bwd_varlen_workspace_size(len(lengths), L, t["total"], H, D),), 0x7F, dtype=torch.uint8,
                    device=cuda_device)
    grads = fa.backward_varlen(d["q"], d["k"], d["v"], o, d["do"], lse, cu, L, causal, scale, deterministic=True,
                               workspace=ws)
    fa.check_device_error()
    _check(t, causal, scale, grads, list(range(H)), f"deterministic dirty workspace D={D} causal={causal}")
