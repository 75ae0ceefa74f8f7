"""Forward parity on the GPU: the sm_100a kernel through the C ABI against
the fp64 oracle on identical seeded 16-bit inputs."""
import math

import numpy as np
import pytest
import torch

import exact_tiled_attention_31_b200 as fa
from exact_tiled_attention_31_b200 import inputs
from oracle import attention as oa
from helpers import check_lse, check_o, f64, to_dev

pytestmark = pytest.mark.gpu


def _fwd(t, causal, scale, dev):
    d = to_dev(t, dev)
    o, lse = fa.forward(d["q"], d["k"], d["v"], causal, scale)
    fa.check_device_error()
    return o, lse


def test_first_config_b1_h2_s256_d64(cuda_device):
    """B=1 H=2 S=256 D=64 bf16, scale 1/8, non-causal: every element."""
    t = inputs.make_dense(1, 2, 256, 64, "bf16", seed=42)
    o, lse = _fwd(t, False, 0.125, cuda_device)
    o_ref, l_ref = oa.attention_forward(t["q"], t["k"], t["v"], 0.125, False)
    check_lse(lse, l_ref, "lse")
    check_o(o, o_ref, "O")


def test_q_zero_gives_mean_of_v(cuda_device):
    """Q = 0 makes every score 0: O is the (prefix) mean of V, LSE = ln(n).
    Independent of the Q K^T product, so it isolates the P V path."""
    for D in (64, 128):
        for causal in (False, True):
            t = inputs.make_dense(1, 2, 300, D, "bf16", seed=7)
            t["q"].zero_()
            o, lse = _fwd(t, causal, 1 / math.sqrt(D), cuda_device)
            v = f64(t["v"])
            n = np.arange(1, 301)[:, None]
            exp_o = np.cumsum(v, axis=2) / n if causal else np.broadcast_to(v.mean(2, keepdims=True), v.shape)
            exp_l = np.log(np.arange(1, 301)) if causal else np.full(300, math.log(300))
            check_o(o, exp_o, f"Q=0 D={D} causal={causal}")
            check_lse(lse, np.broadcast_to(exp_l, (1, 2, 300)), f"Q=0 D={D} causal={causal}")


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("causal", [False, True])
def test_b2_h8_s512_d64(cuda_device, dtype, causal):
    t = inputs.make_dense(2, 8, 512, 64, dtype, seed=42)
    o, lse = _fwd(t, causal, 0.125, cuda_device)
    o_ref, l_ref = oa.attention_forward(t["q"], t["k"], t["v"], 0.125, causal)
    check_lse(lse, l_ref, f"lse {dtype} causal={causal}")
    check_o(o, o_ref, f"O {dtype} causal={causal}")


@pytest.mark.parametrize("S", [1, 17, 127, 128, 129, 255, 256, 257, 383, 640])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_lengths(cuda_device, S, D, causal):
    """Lengths that are not multiples of the 128-row tile, and tiny ones."""
    t = inputs.make_dense(1, 3, S, D, "bf16", seed=S)
    o, lse = _fwd(t, causal, 1 / math.sqrt(D), cuda_device)
    o_ref, l_ref = oa.attention_forward(t["q"], t["k"], t["v"], 1 / math.sqrt(D), causal)
    check_lse(lse, l_ref, f"S={S} D={D} causal={causal}")
    check_o(o, o_ref, f"S={S} D={D} causal={causal}")


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("S", [512, 1024, 2048, 4096])
def test_b1_h32_d128_causal_sweep(cuda_device, S, dtype):
    """B=1 H=32 D=128 causal at the four lengths of the pages' Ascend table.
    Every element up to S=1024; all rows of four heads (first and last
    included) beyond that."""
    t = inputs.make_dense(1, 32, S, 128, dtype, seed=42)
    scale = 1 / math.sqrt(128)
    o, lse = _fwd(t, True, scale, cuda_device)
    if S <= 1024:
        o_ref, l_ref = oa.attention_forward(t["q"], t["k"], t["v"], scale, True)
        check_lse(lse, l_ref, "lse")
        check_o(o, o_ref, "O")
    else:
        heads = [(0, 0), (0, 9), (0, 22), (0, 31)]
        o_ref, l_ref = oa.attention_forward(t["q"], t["k"], t["v"], scale, True, heads=heads)
        sel = [h for _, h in heads]
        check_lse(lse[0, sel], l_ref, "lse")
        check_o(o[0, sel], o_ref, "O")


def test_b1_h32_s32768_d128_sampled_rows(cuda_device):
    """Single long sequence, causal: sampled rows of two heads, computed one
    by one by the oracle."""
    S = 32768
    t = inputs.make_dense(1, 32, S, 128, "bf16", seed=42)
    scale = 1 / math.sqrt(128)
    o, lse = _fwd(t, True, scale, cuda_device)
    rng = np.random.default_rng(0)
    rows = sorted(set([0, 1, 127, 128, 255, 256, 4095, 16384, S - 129, S - 1] +
                      list(rng.integers(0, S, 48))))
    for h in (0, 31):
        o_ref, l_ref = oa.attention_forward_rows(t["q"], t["k"], t["v"], scale, True, 0, h, rows)
        check_lse(lse[0, h, rows], l_ref, f"lse h={h}")
        check_o(o[0, h, rows], o_ref, f"O h={h}")


def test_varlen_packed_batch(cuda_device):
    """32 sequences, lengths uniform in [128, 4096], H=16 D=64 causal, with Q
    and K drawn N(0,1)*8 (scores up to +-64: exercises the running max).
    Every sequence of two heads is checked."""
    t = inputs.make_varlen(32, 128, 4096, 16, 64, "bf16", seed=42, qk_mult=8.0)
    d = to_dev(t, cuda_device)
    o, lse = fa.forward_varlen(d["q"], d["k"], d["v"], d["cu_seqlens"], max(t["lengths"]), True, 0.125)
    fa.check_device_error()
    heads = [0, 15]
    o_ref, l_ref = oa.varlen_forward(t["q"], t["k"], t["v"], t["cu_seqlens"], 0.125, True, heads=heads)
    check_lse(lse[heads], l_ref, "lse")
    check_o(o[heads], o_ref, "O")


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_small_mixed(cuda_device, causal):
    """Short, ragged and single-token sequences in one pack, D=128, fp16."""
    lengths = [1, 5, 128, 129, 300, 17, 256, 2]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T = int(cu[-1])
    g = torch.Generator().manual_seed(3)
    q, k, v = (torch.randn(4, T, 128, generator=g).to(torch.float16) for _ in range(3))
    o, lse = fa.forward_varlen(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device),
                               torch.tensor(cu, device=cuda_device), max(lengths), causal, 0.09)
    fa.check_device_error()
    o_ref, l_ref = oa.varlen_forward(q, k, v, cu, 0.09, causal)
    check_lse(lse, l_ref, "lse")
    check_o(o, o_ref, "O")


def test_gpu_invariants(cuda_device):
    """Dominant score selects its V row; permuting K/V rows together leaves a
    non-causal result unchanged (up to summation order)."""
    S, D = 384, 128
    t = inputs.make_dense(1, 1, S, D, "bf16", seed=11)
    q = torch.zeros(1, 1, S, D)
    q[..., 0] = 1.0
    k = t["k"].float() * 0.01
    k[0, 0, 200, 0] = 64.0
    t2 = {"q": q.bfloat16(), "k": k.bfloat16(), "v": t["v"]}
    o, _ = _fwd(t2, False, 1.0, cuda_device)
    np.testing.assert_allclose(f64(o)[0, 0], np.broadcast_to(f64(t["v"])[0, 0, 200], (S, D)), atol=1e-2)
    perm = torch.randperm(S, generator=torch.Generator().manual_seed(1))
    o1, l1 = _fwd(t, False, 0.1, cuda_device)
    o2, l2 = _fwd({"q": t["q"], "k": t["k"][:, :, perm], "v": t["v"][:, :, perm]}, False, 0.1, cuda_device)
    check_o(o2, o1, "permuted K/V")
    check_lse(l2, l1, "permuted K/V")


def test_causal_differs_from_full(cuda_device):
    """A dropped causal mask must show ("ops-transformer里的FlashAttention", 坑二)."""
    t = inputs.make_dense(1, 2, 256, 64, "bf16", seed=5)
    o1, _ = _fwd(t, False, 0.125, cuda_device)
    o2, _ = _fwd(t, True, 0.125, cuda_device)
    assert (o1.float() - o2.float()).abs().max().item() > 0.1
    # the last row sees every key either way
    torch.testing.assert_close(o1[:, :, -1].float(), o2[:, :, -1].float(), atol=1e-2, rtol=0)


def test_timeout_path_reports_and_recovers(cuda_device):
    """A bounded wait that runs out records FA_ERR_TIMEOUT (no fault, no
    hang); the error word is cleared by the check and the context keeps
    working for the next call."""
    st = torch.cuda.current_stream().cuda_stream
    assert fa.fa_selftest_timeout(st) == fa.api.FA_OK
    assert fa.fa_check_device_error(st) == fa.api.FA_ERR_TIMEOUT
    assert fa.fa_check_device_error(st) == fa.api.FA_OK  # cleared
    t = inputs.make_dense(1, 2, 256, 64, "bf16", seed=42)
    d = to_dev(t, cuda_device)
    o, lse = fa.forward(d["q"], d["k"], d["v"], False, 0.125)
    fa.check_device_error()
    o_ref, l_ref = oa.attention_forward(t["q"], t["k"], t["v"], 0.125, False)
    check_o(o, o_ref, "O after a timeout")
    check_lse(lse, l_ref, "LSE after a timeout")
