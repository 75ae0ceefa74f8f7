"""Dropout parity on the GPU for packed variable-length batches:
fa_fwd_varlen_dropout / fa_bwd_varlen_dropout against the fp64 oracle, in
which sequence s of a pack takes the mask of batch index s of a dense batch.

* the keep mask itself, bit for bit (Q = 0, V = I as in the dense test);
* O, LSE, dQ, dK, dV on mixed lengths within the stated tolerances;
* a pack of equal lengths drops exactly what the dense batch drops, so its
  outputs equal the dense call's bit for bit (deterministic backward)."""
import math

import numpy as np
import pytest
import torch

import exact_tiled_attention_31_b200 as fa
from oracle import attention as oa
from helpers import check_grad, check_lse, check_o, f64, to_dev

pytestmark = pytest.mark.gpu


def _pack(lengths, H, D, dtype, seed):
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T = int(cu[-1])
    g = torch.Generator().manual_seed(seed)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float16
    out = {k: torch.randn(H, T, D, generator=g).to(dt) for k in ("q", "k", "v", "do")}
    out.update(lengths=list(lengths), cu_seqlens=torch.tensor(cu), total=T)
    return out


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_forward_mask_is_the_oracle_mask(cuda_device, causal):
    """Each sequence's O is nonzero exactly at its own (s * H + h) mask."""
    lengths, H, D, p, seed, offset = [128, 37, 128, 5], 3, 128, 0.4, 99, 3
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T = int(cu[-1])
    dev = cuda_device
    q = torch.zeros(H, T, D, dtype=torch.bfloat16, device=dev)
    k = torch.randn(H, T, D, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16).to(dev)
    v = torch.zeros(H, T, D, dtype=torch.bfloat16)
    for a, b in zip(cu[:-1], cu[1:]):
        v[:, a:b, : b - a] = torch.eye(b - a, dtype=torch.bfloat16)
    v = v.to(dev)
    o, _ = fa.forward_varlen(q, k, v, torch.tensor(cu).to(dev), max(lengths), causal, 0.1, dropout_p=p, seed=seed,
                             offset=offset)
    fa.check_device_error()
    got = f64(o) != 0
    for s, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        L = b - a
        for h in range(H):
            want = oa.dropout_keep(s * H + h, np.arange(L), np.arange(L), p, seed, offset)
            if causal:
                want &= np.tril(np.ones((L, L), dtype=bool))
            assert np.array_equal(got[h, a:b, :L], want), f"sequence {s} head {h}"


@pytest.mark.parametrize("lengths,H,D,dtype,causal,p", [
    ([1, 5, 128, 129, 300, 17, 256, 2], 4, 128, "fp16", True, 0.2),
    ([1, 5, 128, 129, 300, 17, 256, 2], 4, 128, "bf16", False, 0.3),
    ([200, 64, 513, 1, 130], 2, 64, "bf16", True, 0.1),
    ([200, 64, 513, 1, 130], 2, 64, "fp16", False, 0.5),
])
def test_varlen_dropout_matches_oracle(cuda_device, lengths, H, D, dtype, causal, p):
    t = _pack(lengths, H, D, dtype, seed=sum(lengths) + D)
    scale, seed, offset = 1.0 / math.sqrt(D), 31337, 4
    d = to_dev(t, cuda_device)
    cu = t["cu_seqlens"].to(cuda_device)
    L = max(lengths)
    o, lse = fa.forward_varlen(d["q"], d["k"], d["v"], cu, L, causal, scale, dropout_p=p, seed=seed, offset=offset)
    grads = fa.backward_varlen(d["q"], d["k"], d["v"], o, d["do"], lse, cu, L, causal, scale, dropout_p=p, seed=seed,
                               offset=offset)
    fa.check_device_error()
    what = f"packed dropout {lengths} H{H} D{D} {dtype} causal={causal} p={p}"
    ro, rl = oa.varlen_forward_dropout(t["q"], t["k"], t["v"], t["cu_seqlens"], scale, causal, p, seed, offset)
    check_o(o, ro, f"O {what}")
    check_lse(lse, rl, f"LSE {what}")
    ref = oa.varlen_backward_dropout(t["q"], t["k"], t["v"], t["do"], t["cu_seqlens"], scale, causal, p, seed, offset)
    for g, r, name in zip(grads, ref, ("dQ", "dK", "dV")):
        check_grad(g, r, f"{name} {what}")


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_dropout_equal_lengths_is_the_dense_batch(cuda_device, causal):
    B, H, S, D, p = 3, 2, 300, 128, 0.25
    t = _pack([S] * B, H, D, "bf16", seed=8)
    d = to_dev(t, cuda_device)
    cu = t["cu_seqlens"].to(cuda_device)
    kw = dict(dropout_p=p, seed=77, offset=6)
    o_v, lse_v = fa.forward_varlen(d["q"], d["k"], d["v"], cu, S, causal, 0.09, **kw)
    gv = fa.backward_varlen(d["q"], d["k"], d["v"], o_v, d["do"], lse_v, cu, S, causal, 0.09, deterministic=True, **kw)
    dense = {k: d[k].view(H, B, S, D).transpose(0, 1).contiguous() for k in ("q", "k", "v", "do")}
    o_d, lse_d = fa.forward(dense["q"], dense["k"], dense["v"], causal, 0.09, **kw)
    gd = fa.backward(dense["q"], dense["k"], dense["v"], o_d, dense["do"], lse_d, causal, 0.09, deterministic=True,
                     **kw)
    fa.check_device_error()
    assert torch.equal(o_v, o_d.transpose(0, 1).reshape(H, B * S, D))
    assert torch.equal(lse_v, lse_d.transpose(0, 1).reshape(H, B * S))
    for a, b, name in zip(gv, gd, ("dQ", "dK", "dV")):
        assert torch.equal(a, b.transpose(0, 1).reshape(H, B * S, D)), name


def test_varlen_dropout_zero_is_the_plain_path(cuda_device):
    t = _pack([300, 1, 777], 2, 128, "bf16", seed=9)
    d = to_dev(t, cuda_device)
    cu = t["cu_seqlens"].to(cuda_device)
    o0, l0 = fa.forward_varlen(d["q"], d["k"], d["v"], cu, 777, True)
    o1 = torch.empty_like(o0)
    l1 = torch.empty_like(l0)
    st = fa.fa_fwd_varlen_dropout(d["q"].data_ptr(), d["k"].data_ptr(), d["v"].data_ptr(), o1.data_ptr(),
                                  l1.data_ptr(), cu.data_ptr(), 3, 777, t["total"], 2, 128, 1 / math.sqrt(128), 1, 0,
                                  0.0, 5, 5, torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    assert torch.equal(o0, o1) and torch.equal(l0, l1)
