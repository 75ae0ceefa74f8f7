"""Decode parity on the GPU: fa_decode (split-KV over a KV cache, with the
(O, LSE) merge and grouped-query heads) against the fp64 oracle's
decode_forward, element by element on O and LSE."""
import math

import numpy as np
import pytest
import torch

import exact_tiled_attention_31_b200 as fa
from exact_tiled_attention_31_b200 import inputs
from oracle import attention as oa
from helpers import check_lse, check_o, f64

pytestmark = pytest.mark.gpu


def _run(t, dev, n_splits=None, scale=None):
    q, k, v = (t[x].to(dev) for x in ("q", "k", "v"))
    lens = t["seq_lens"].to(dev)
    o, lse = fa.decode(q, k, v, lens, scale=scale, n_splits=n_splits)
    fa.check_device_error()
    return o, lse


def _ref(t, scale, batches=None):
    lens = t["seq_lens"].numpy()
    bs = range(len(lens)) if batches is None else batches
    o, lse = oa.decode_forward(t["q"][list(bs)], t["k"][list(bs)], t["v"][list(bs)], lens[list(bs)], scale)
    return o, lse


@pytest.mark.parametrize("Hq,Hkv,D,dtype,n_splits", [
    (32, 8, 128, "bf16", None),    # GQA, group 4, library's split choice
    (32, 32, 128, "bf16", 8),      # multi-head
    (16, 1, 64, "fp16", 32),       # multi-query, group 16 (the largest)
    (12, 3, 64, "bf16", 1),        # one split: the merge of a single part
    (10, 2, 128, "fp16", 5),       # group 5: padded query rows
])
def test_decode_matches_oracle(cuda_device, Hq, Hkv, D, dtype, n_splits):
    t = inputs.make_decode(4, Hq, Hkv, 1000, D, dtype, seed=11)
    scale = 1.0 / math.sqrt(D)
    o, lse = _run(t, cuda_device, n_splits)
    ro, rl = _ref(t, scale)
    check_o(o, ro, f"decode Hq{Hq} Hkv{Hkv} D{D} {dtype} splits {n_splits}")
    check_lse(lse, rl, "decode LSE")


@pytest.mark.parametrize("B,Hq,Hkv,D,dtype,n_splits", [
    (4, 16, 4, 64, "bf16", 2),      # D = 64 splits merged in-kernel (2-CTA clusters, 32 CTAs)
    (3, 8, 8, 64, "fp16", 4),       # D = 64, 4-CTA clusters
    (40, 8, 4, 128, "bf16", 4),     # 4 splits over 160 CTAs (more than one wave): merge kernel
])
def test_decode_merge_paths(cuda_device, B, Hq, Hkv, D, dtype, n_splits):
    t = inputs.make_decode(B, Hq, Hkv, 600, D, dtype, seed=B + D)
    o, lse = _run(t, cuda_device, n_splits)
    ro, rl = _ref(t, 1.0 / math.sqrt(D))
    check_o(o, ro, f"decode merge path B{B} Hq{Hq} Hkv{Hkv} D{D} splits {n_splits}")
    check_lse(lse, rl, "decode merge path LSE")


def test_decode_ragged_lengths_and_edges(cuda_device):
    """Lengths at and around the 32-key tile, a single key, the full cache,
    a length past the cache (clamped to L_max) and an empty sequence
    (O = 0, LSE = -inf)."""
    L, D = 300, 128
    lens = [1, 31, 32, 33, 63, 64, 65, 255, 299, 300, 1000, 0]
    t = inputs.make_decode(len(lens), 8, 2, L, D, "bf16", seed=5)
    t["seq_lens"] = torch.tensor(lens, dtype=torch.int32)
    o, lse = _run(t, cuda_device, n_splits=3, scale=0.1)
    clamped = dict(t, seq_lens=torch.tensor([min(x, L) for x in lens], dtype=torch.int32))
    live = [b for b, x in enumerate(lens) if x > 0]
    ro, rl = _ref(clamped, 0.1, live)
    check_o(o[live], ro, "ragged lengths")
    check_lse(lse[live], rl, "ragged lengths LSE")
    empty = lens.index(0)
    assert torch.all(o[empty] == 0)
    assert torch.all(torch.isneginf(lse[empty]))


def test_decode_never_reads_past_length(cuda_device):
    """Cache rows at or past seq_lens[b] hold NaN; any read of them would
    reach O through 0 * NaN."""
    t = inputs.make_decode(3, 16, 4, 700, 64, "bf16", seed=8)
    t["seq_lens"] = torch.tensor([700, 333, 65], dtype=torch.int32)
    ro, rl = _ref(t, 0.125)
    for b, n in enumerate(t["seq_lens"].tolist()):
        t["k"][b, :, n:] = float("nan")
        t["v"][b, :, n:] = float("nan")
    for n_splits in (1, 7):
        o, lse = _run(t, cuda_device, n_splits=n_splits, scale=0.125)
        check_o(o, ro, f"poisoned tail, splits {n_splits}")
        check_lse(lse, rl, "poisoned tail LSE")


def test_decode_split_count_invariance(cuda_device):
    """The answer does not depend on how the cache is cut (only rounding)."""
    t = inputs.make_decode(2, 8, 8, 4096, 128, "bf16", seed=21)
    outs = [_run(t, cuda_device, n_splits=n) for n in (1, 2, 16, 64, 128)]
    ro, rl = _ref(t, 1.0 / math.sqrt(128))
    for o, lse in outs:
        check_o(o, ro, "split invariance")
        check_lse(lse, rl, "split invariance LSE")
    base = f64(outs[0][0])
    for o, _ in outs[1:]:
        assert np.abs(f64(o) - base).max() <= 2e-2


def test_decode_large_scores(cuda_device):
    """Q and K scaled by 8 (scores up to a few hundred): exact maximum and
    the merge's rescaling must keep every exponent at or below zero."""
    t = inputs.make_decode(2, 8, 2, 2000, 128, "bf16", seed=4)
    t["q"] = (t["q"].float() * 8).to(torch.bfloat16)
    t["k"] = (t["k"].float() * 8).to(torch.bfloat16)
    o, lse = _run(t, cuda_device, n_splits=9, scale=0.125)
    ro, rl = _ref(t, 0.125)
    check_o(o, ro, "large scores")
    check_lse(lse, rl, "large scores LSE")


def test_decode_full_size_sampled(cuda_device):
    """The benchmark's configuration: B8 Hq32 Hkv8 L8192 D128 bf16, every
    cache full, the library's split choice; two sequences are checked against
    the oracle head by head."""
    t = inputs.make_decode(8, 32, 8, 8192, 128, "bf16", seed=42)
    t["seq_lens"] = torch.full((8,), 8192, dtype=torch.int32)
    o, lse = _run(t, cuda_device)
    ro, rl = _ref(t, 1.0 / math.sqrt(128), [0, 7])
    check_o(o[[0, 7]], ro, "full size")
    check_lse(lse[[0, 7]], rl, "full size LSE")


@pytest.mark.parametrize("B,Hq,Hkv,L,D,dtype", [
    (4, 32, 8, 1000, 128, "bf16"),   # caches of 32 tiles over 128 CTAs: one cache per several CTAs
    (40, 8, 4, 600, 128, "bf16"),    # 160 caches of 19 tiles over 148 CTAs: runs that span two caches
    (3, 16, 1, 700, 64, "fp16"),     # multi-query, group 16, D = 64
    (2, 10, 2, 33, 128, "fp16"),     # two tiles per cache, group 5 (padded rows): fewer tiles than SMs
])
def test_decode_balanced_matches_oracle(cuda_device, B, Hq, Hkv, L, D, dtype):
    """Balanced mode (n_splits = 0): the caches' 32-key tiles dealt out evenly
    over one CTA per SM, each cache's parts merged by their LSE."""
    t = inputs.make_decode(B, Hq, Hkv, L, D, dtype, seed=B * L + D)
    o, lse = _run(t, cuda_device, n_splits=0)
    ro, rl = _ref(t, 1.0 / math.sqrt(D))
    check_o(o, ro, f"balanced B{B} Hq{Hq} Hkv{Hkv} L{L} D{D} {dtype}")
    check_lse(lse, rl, "balanced LSE")


def test_decode_balanced_ragged_and_poisoned(cuda_device):
    """Balanced mode over ragged lengths (empty, single key, tile edges, past
    the cache) with every cache row at or past a length set to NaN."""
    L, D = 300, 128
    lens = [1, 31, 32, 33, 64, 65, 255, 299, 300, 1000, 0, 7]
    t = inputs.make_decode(len(lens), 8, 2, L, D, "bf16", seed=6)
    t["seq_lens"] = torch.tensor(lens, dtype=torch.int32)
    clamped = [min(x, L) for x in lens]
    live = [b for b, x in enumerate(lens) if x > 0]
    ro, rl = _ref(dict(t, seq_lens=torch.tensor(clamped, dtype=torch.int32)), 0.1, live)
    for b, n in enumerate(clamped):
        t["k"][b, :, n:] = float("nan")
        t["v"][b, :, n:] = float("nan")
    o, lse = _run(t, cuda_device, n_splits=0, scale=0.1)
    check_o(o[live], ro, "balanced ragged")
    check_lse(lse[live], rl, "balanced ragged LSE")
    empty = lens.index(0)
    assert torch.all(o[empty] == 0)
    assert torch.all(torch.isneginf(lse[empty]))


def test_decode_long_context_sampled(cuda_device):
    """One sequence with a 32768-key cache (B1 Hq32 Hkv8 D128 bf16), the
    library's choice of cut and balanced mode, checked against the oracle."""
    t = inputs.make_decode(1, 32, 8, 32768, 128, "bf16", seed=3)
    t["seq_lens"] = torch.full((1,), 32768, dtype=torch.int32)
    ro, rl = _ref(t, 1.0 / math.sqrt(128))
    for n_splits in (None, 0):
        o, lse = _run(t, cuda_device, n_splits=n_splits)
        check_o(o, ro, f"long context, splits {n_splits}")
        check_lse(lse, rl, "long context LSE")
