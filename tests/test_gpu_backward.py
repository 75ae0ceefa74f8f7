"""Backward parity on the GPU: dQ, dK, dV from the sm_100a kernels (P rebuilt
from the forward's LSE) against the fp64 oracle's textbook gradients."""
import math

import numpy as np
import pytest
import torch

import exact_tiled_attention_31_b200 as fa
from exact_tiled_attention_31_b200 import inputs
from oracle import attention as oa
from helpers import check_grad, check_lse, check_o, f64, to_dev

pytestmark = pytest.mark.gpu


def _fwd_bwd(t, causal, scale, dev, deterministic=False):
    d = to_dev(t, dev)
    o, lse = fa.forward(d["q"], d["k"], d["v"], causal, scale)
    dq, dk, dv = fa.backward(d["q"], d["k"], d["v"], o, d["do"], lse, causal, scale, deterministic)
    fa.check_device_error()
    return o, lse, dq, dk, dv


def _check_all(t, causal, scale, res, heads=None, what=""):
    o, lse, dq, dk, dv = res
    if heads is None:
        gq, gk, gv = oa.attention_backward(t["q"], t["k"], t["v"], t["do"], scale, causal)
        sel = (slice(None), slice(None))
    else:
        gq, gk, gv = oa.attention_backward(t["q"], t["k"], t["v"], t["do"], scale, causal, heads=heads)
        sel = ([b for b, _ in heads], [h for _, h in heads])
    check_grad(dq[sel], gq, f"dQ {what}")
    check_grad(dk[sel], gk, f"dK {what}")
    check_grad(dv[sel], gv, f"dV {what}")


def test_bwd_first_config(cuda_device):
    t = inputs.make_dense(1, 2, 256, 64, "bf16", seed=42, with_do=True)
    _check_all(t, False, 0.125, _fwd_bwd(t, False, 0.125, cuda_device), what="B1 H2 S256 D64")


def test_bwd_q_zero_dv_closed_form(cuda_device):
    """Q = 0: every visible P_ij = 1/n_i, so dV_j = sum_{i sees j} dO_i / n_i."""
    S, D = 300, 128
    t = inputs.make_dense(1, 1, S, D, "bf16", seed=9, with_do=True)
    t["q"].zero_()
    _, _, _, _, dv = _fwd_bwd(t, True, 1 / math.sqrt(D), cuda_device)
    do = f64(t["do"])[0, 0]
    expect = np.cumsum((do / np.arange(1, S + 1)[:, None])[::-1], axis=0)[::-1]
    check_grad(dv[0, 0], expect, "dV (Q=0, causal)")


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_b2_h8_s512_d64(cuda_device, dtype, causal):
    t = inputs.make_dense(2, 8, 512, 64, dtype, seed=42, with_do=True)
    _check_all(t, causal, 0.125, _fwd_bwd(t, causal, 0.125, cuda_device), what=f"{dtype} causal={causal}")


@pytest.mark.parametrize("S", [1, 17, 129, 255, 383])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_ragged(cuda_device, S, D, causal):
    t = inputs.make_dense(1, 2, S, D, "bf16", seed=S + D, with_do=True)
    _check_all(t, causal, 1 / math.sqrt(D), _fwd_bwd(t, causal, 1 / math.sqrt(D), cuda_device),
               what=f"S={S} D={D} causal={causal}")


def test_bwd_b1_h32_s4096_d128_causal(cuda_device):
    """The benchmarked workload: all rows of four heads."""
    t = inputs.make_dense(1, 32, 4096, 128, "bf16", seed=42, with_do=True)
    scale = 1 / math.sqrt(128)
    res = _fwd_bwd(t, True, scale, cuda_device)
    _check_all(t, True, scale, res, heads=[(0, 0), (0, 13), (0, 27), (0, 31)], what="B1 H32 S4096")


def test_bwd_training_b4_h16_s8192_d128(cuda_device):
    """Training shape, causal: all rows of four (b, h) heads."""
    t = inputs.make_dense(4, 16, 8192, 128, "bf16", seed=42, with_do=True)
    scale = 1 / math.sqrt(128)
    res = _fwd_bwd(t, True, scale, cuda_device)
    heads = [(0, 0), (1, 7), (2, 12), (3, 15)]
    o_ref, l_ref = oa.attention_forward(t["q"], t["k"], t["v"], scale, True, heads=heads)
    sel = ([b for b, _ in heads], [h for _, h in heads])
    check_o(res[0][sel], o_ref, "O")
    check_lse(res[1][sel], l_ref, "lse")
    _check_all(t, True, scale, res, heads=heads, what="B4 H16 S8192")


def test_bwd_deterministic_is_bitwise_repeatable(cuda_device):
    t = inputs.make_dense(2, 4, 1024, 128, "bf16", seed=1, with_do=True)
    d = to_dev(t, cuda_device)
    o, lse = fa.forward(d["q"], d["k"], d["v"], True, 0.088)
    runs = [fa.backward(d["q"], d["k"], d["v"], o, d["do"], lse, True, 0.088, deterministic=True) for _ in range(3)]
    fa.check_device_error()
    for r in runs[1:]:
        for a, b in zip(runs[0], r):
            assert torch.equal(a, b)
    nd = fa.backward(d["q"], d["k"], d["v"], o, d["do"], lse, True, 0.088, deterministic=False)
    for a, b, name in zip(runs[0], nd, ("dQ", "dK", "dV")):
        check_grad(b, a, f"{name} atomic vs ordered")


@pytest.mark.parametrize("S", [1, 17, 129, 255, 383])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_deterministic_on_dirty_workspace_matches_oracle(cuda_device, S, D, causal):
    """Deterministic mode on a workspace full of 0x7F bytes (3.4e38 as fp32),
    ragged lengths, one tile and several: both dQ accumulators must be
    cleared inside the call (the second one holds the odd key tiles, and no
    key tile at all reaches it for query tile 0 under the causal mask), so
    no byte from before the call may reach dQ."""
    B, H = 2, 2
    t = inputs.make_dense(B, H, S, D, "bf16", seed=S * D + causal, with_do=True)
    d = to_dev(t, cuda_device)
    scale = 1 / math.sqrt(D)
    o, lse = fa.forward(d["q"], d["k"], d["v"], causal, scale)
    ws = torch.full((fa.fa_bwd_workspace_size(B, H, S, D),), 0x7F, dtype=torch.uint8, device=cuda_device)
    g = fa.backward(d["q"], d["k"], d["v"], o, d["do"], lse, causal, scale, deterministic=True, workspace=ws)
    fa.check_device_error()
    _check_all(t, causal, scale, (o, lse, *g), what=f"deterministic S={S} D={D} causal={causal}")


def test_bwd_workspace_reuse_and_dirty(cuda_device):
    """The workspace may hold anything on entry (it is cleared inside)."""
    t = inputs.make_dense(1, 2, 640, 64, "fp16", seed=4, with_do=True)
    d = to_dev(t, cuda_device)
    o, lse = fa.forward(d["q"], d["k"], d["v"], True, 0.125)
    ws = torch.full((fa.fa_bwd_workspace_size(1, 2, 640, 64),), 0x7F, dtype=torch.uint8, device=cuda_device)
    a = fa.backward(d["q"], d["k"], d["v"], o, d["do"], lse, True, 0.125, workspace=ws)
    b = fa.backward(d["q"], d["k"], d["v"], o, d["do"], lse, True, 0.125, workspace=ws)
    fa.check_device_error()
    for x, y, name in zip(a, b, ("dQ", "dK", "dV")):
        check_grad(y, x, name)
    _check_all(t, True, 0.125, (o, lse, *a), what="dirty workspace")


def test_bwd_split_launches_equal_fa_bwd(cuda_device):
    """fa_bwd_preprocess + fa_bwd_main + fa_bwd_finish (the launches bench.py
    times one by one) give exactly what fa_bwd gives (deterministic mode)."""
    B, H, S, D = 1, 3, 520, 128
    t = inputs.make_dense(B, H, S, D, "bf16", seed=8, with_do=True)
    d = to_dev(t, cuda_device)
    o, lse = fa.forward(d["q"], d["k"], d["v"], True, 0.088)
    ref = fa.backward(d["q"], d["k"], d["v"], o, d["do"], lse, True, 0.088, deterministic=True)
    nb = fa.fa_bwd_workspace_size(B, H, S, D)
    ws = torch.empty(nb, dtype=torch.uint8, device=cuda_device)
    dq, dk, dv = (torch.empty_like(d["q"]) for _ in range(3))
    st = torch.cuda.current_stream().cuda_stream
    dt = fa.api.FA_BF16
    assert fa.fa_bwd_preprocess(o.data_ptr(), d["do"].data_ptr(), lse.data_ptr(), B, H, S, D, dt, ws.data_ptr(), nb,
                                st) == 0
    assert fa.fa_bwd_main(d["q"].data_ptr(), d["k"].data_ptr(), d["v"].data_ptr(), d["do"].data_ptr(), dk.data_ptr(),
                          dv.data_ptr(), B, H, S, D, 0.088, True, dt, True, ws.data_ptr(), nb, st) == 0
    assert fa.fa_bwd_finish(dq.data_ptr(), B, H, S, D, 0.088, dt, True, ws.data_ptr(), nb, st) == 0
    fa.check_device_error()
    for a, b, name in zip((dq, dk, dv), ref, ("dQ", "dK", "dV")):
        assert torch.equal(a, b), name


@pytest.mark.parametrize("det_main", [False, True])
def test_bwd_split_mode_mismatch_is_reported(cuda_device, det_main):
    """fa_bwd_finish told the other deterministic mode than fa_bwd_main ran
    in records an argument error (read back as FA_ERR_INVALID_ARG, which also
    clears it); the same calls with matching modes record none."""
    B, H, S, D = 1, 2, 300, 64
    t = inputs.make_dense(B, H, S, D, "bf16", seed=9, with_do=True)
    d = to_dev(t, cuda_device)
    o, lse = fa.forward(d["q"], d["k"], d["v"], False, 0.125)
    nb = fa.fa_bwd_workspace_size(B, H, S, D)
    ws = torch.empty(nb, dtype=torch.uint8, device=cuda_device)
    dq, dk, dv = (torch.empty_like(d["q"]) for _ in range(3))
    st = torch.cuda.current_stream().cuda_stream
    dt = fa.api.FA_BF16
    fa.check_device_error()
    for det_finish, want in ((not det_main, fa.api.FA_ERR_INVALID_ARG), (det_main, fa.api.FA_OK)):
        assert fa.fa_bwd_preprocess(o.data_ptr(), d["do"].data_ptr(), lse.data_ptr(), B, H, S, D, dt, ws.data_ptr(),
                                    nb, st) == 0
        assert fa.fa_bwd_main(d["q"].data_ptr(), d["k"].data_ptr(), d["v"].data_ptr(), d["do"].data_ptr(),
                              dk.data_ptr(), dv.data_ptr(), B, H, S, D, 0.125, False, dt, det_main, ws.data_ptr(), nb,
                              st) == 0
        assert fa.fa_bwd_finish(dq.data_ptr(), B, H, S, D, 0.125, dt, det_finish, ws.data_ptr(), nb, st) == 0
        assert fa.fa_check_device_error(st) == want
