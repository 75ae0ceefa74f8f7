"""Seeded synthetic inputs shared by the CUDA path, the tests and the bench.

This module only draws random numbers and rounds them to the storage dtype.
It holds none of the attention arithmetic, so both the fp64 oracle and the
CUDA kernels can be fed from it without sharing any of the method's code.

Draw convention (the pages' own check in "From Self-Attention to
FlashAttention", §二, seeds the generator with 42 and draws Q, K, V with
``randn``):

* one CPU ``torch.Generator`` seeded with ``seed``;
* varlen sequence lengths are drawn first, uniform in ``[lo, hi]``
  (inclusive);
* then Q, K, V and (for training) dO are drawn in that order as fp32
  ``N(0, 1)``, Q and K optionally multiplied by ``qk_mult`` (a power of two,
  so the product is exact), and finally rounded to nearest into bf16/fp16.

Layouts: dense tensors are ``[B, H, S, D]`` contiguous; packed varlen
tensors are ``[H, T, D]`` contiguous with ``T = sum(lengths)`` and
``cu_seqlens`` int32 ``[nseq + 1]``.
"""
from __future__ import annotations

import torch

_DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16}


def torch_dtype(name: str) -> torch.dtype:
    """Map ``"bf16"``/``"fp16"`` to the torch storage dtype."""
    try:
        return _DTYPES[name]
    except KeyError as exc:  # pragma: no cover - programming error
        raise ValueError(f"unsupported dtype {name!r}") from exc


def _draw(gen: torch.Generator, shape, mult: float, dtype: torch.dtype) -> torch.Tensor:
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if mult != 1.0:
        x.mul_(mult)
    return x.to(dtype)


def make_dense(B: int, H: int, S: int, D: int, dtype: str = "bf16", seed: int = 42,
               qk_mult: float = 1.0, with_do: bool = False) -> dict:
    """Q, K, V (and dO) as CPU tensors of shape [B, H, S, D] in ``dtype``."""
    gen = torch.Generator().manual_seed(seed)
    dt = torch_dtype(dtype)
    out = {
        "q": _draw(gen, (B, H, S, D), qk_mult, dt),
        "k": _draw(gen, (B, H, S, D), qk_mult, dt),
        "v": _draw(gen, (B, H, S, D), 1.0, dt),
    }
    if with_do:
        out["do"] = _draw(gen, (B, H, S, D), 1.0, dt)
    return out


def make_varlen(nseq: int, lo: int, hi: int, H: int, D: int, dtype: str = "bf16",
                seed: int = 42, qk_mult: float = 1.0, with_do: bool = False) -> dict:
    """A packed batch of ``nseq`` sequences with lengths uniform in [lo, hi].

    Returns ``lengths`` (int64 list), ``cu_seqlens`` (int32 CPU tensor of
    ``nseq + 1`` offsets), and Q, K, V (and dO) of shape [H, T, D].
    """
    gen = torch.Generator().manual_seed(seed)
    lengths = torch.randint(lo, hi + 1, (nseq,), generator=gen, dtype=torch.int64)
    cu = torch.zeros(nseq + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(lengths, 0)
    T = int(cu[-1])
    dt = torch_dtype(dtype)
    out = {
        "lengths": [int(x) for x in lengths],
        "cu_seqlens": cu.to(torch.int32),
        "total": T,
        "q": _draw(gen, (H, T, D), qk_mult, dt),
        "k": _draw(gen, (H, T, D), qk_mult, dt),
        "v": _draw(gen, (H, T, D), 1.0, dt),
    }
    if with_do:
        out["do"] = _draw(gen, (H, T, D), 1.0, dt)
    return out


def make_decode(B: int, Hq: int, Hkv: int, L: int, D: int, dtype: str = "bf16", seed: int = 42,
                lo: int = 1) -> dict:
    """Decode inputs: ``seq_lens`` int32 [B] drawn first, uniform in [lo, L];
    then q [B, Hq, D] and the caches k, v [B, Hkv, L, D] as fp32 N(0, 1)
    rounded to ``dtype`` (cache rows past a sequence's length hold values too;
    they must not be read)."""
    gen = torch.Generator().manual_seed(seed)
    lens = torch.randint(lo, L + 1, (B,), generator=gen, dtype=torch.int64)
    dt = torch_dtype(dtype)
    return {
        "seq_lens": lens.to(torch.int32),
        "q": _draw(gen, (B, Hq, D), 1.0, dt),
        "k": _draw(gen, (B, Hkv, L, D), 1.0, dt),
        "v": _draw(gen, (B, Hkv, L, D), 1.0, dt),
    }
