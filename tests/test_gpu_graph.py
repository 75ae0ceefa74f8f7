"""The library's calls inside a CUDA graph: a captured forward + backward
(deterministic, so bit-comparable), dropout step and decode step replay to
exactly what the same calls give when run directly, also after the inputs
are rewritten in place between replays (the graph reads the buffers, it does
not freeze their contents)."""
import math

import pytest
import torch

import exact_tiled_attention_31_b200 as fa
from exact_tiled_attention_31_b200 import inputs

pytestmark = pytest.mark.gpu


def _capture(fn):
    # warm up on a side stream first (library set-up, lazy allocations)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(2):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


@pytest.mark.parametrize("dropout_p", [0.0, 0.2])
def test_forward_backward_graph_replays_bit_exactly(cuda_device, dropout_p):
    B, H, S, D = 1, 4, 1000, 128
    scale = 1.0 / math.sqrt(D)
    dev = cuda_device
    bufs = {k: v.to(dev) for k, v in inputs.make_dense(B, H, S, D, "bf16", seed=1, with_do=True).items()
            if isinstance(v, torch.Tensor)}
    q, k, v, do = (bufs[x] for x in ("q", "k", "v", "do"))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, S), device=dev, dtype=torch.float32)
    grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, S, D), device=dev, dtype=torch.uint8)
    kw = dict(dropout_p=dropout_p, seed=11, offset=3) if dropout_p else {}

    def step():
        fa.forward(q, k, v, True, scale, out=o, lse=lse, **kw)
        fa.backward(q, k, v, o, do, lse, True, scale, deterministic=True, workspace=ws, out=grads, **kw)

    g = _capture(step)
    for seed in (2, 3):
        fresh = inputs.make_dense(B, H, S, D, "bf16", seed=seed, with_do=True)
        for name in ("q", "k", "v", "do"):
            bufs[name].copy_(fresh[name].to(dev))
        g.replay()
        torch.cuda.synchronize()
        fa.check_device_error()
        d = {name: fresh[name].to(dev) for name in ("q", "k", "v", "do")}
        o_ref, lse_ref = fa.forward(d["q"], d["k"], d["v"], True, scale, **kw)
        g_ref = fa.backward(d["q"], d["k"], d["v"], o_ref, d["do"], lse_ref, True, scale, deterministic=True, **kw)
        fa.check_device_error()
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
        for a, b, name in zip(grads, g_ref, ("dQ", "dK", "dV")):
            assert torch.equal(a, b), name


@pytest.mark.parametrize("n_splits", [1, 2, 8, 0])  # 0: balanced mode
def test_decode_graph_replays_bit_exactly(cuda_device, n_splits):
    B, Hq, Hkv, L, D = 4, 16, 4, 2048, 128
    dev = cuda_device
    t = inputs.make_decode(B, Hq, Hkv, L, D, "bf16", seed=5)
    q, kc, vc = (t[x].to(dev) for x in ("q", "k", "v"))
    lens = t["seq_lens"].to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq), device=dev, dtype=torch.float32)
    ws = torch.empty(max(1, fa.fa_decode_workspace_size(B, Hq, n_splits, D)), device=dev, dtype=torch.uint8)

    g = _capture(lambda: fa.decode(q, kc, vc, lens, n_splits=n_splits, out=o, lse=lse, workspace=ws))
    fresh = inputs.make_decode(B, Hq, Hkv, L, D, "bf16", seed=6)
    q.copy_(fresh["q"].to(dev))
    lens.copy_(fresh["seq_lens"].to(dev))
    g.replay()
    torch.cuda.synchronize()
    fa.check_device_error()
    o_ref, lse_ref = fa.decode(q, kc, vc, lens, n_splits=n_splits)
    fa.check_device_error()
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
