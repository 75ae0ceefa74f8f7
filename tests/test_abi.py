"""CPU-side checks of the C ABI: the library loads without a GPU, exports
every function include/fa.h declares, and rejects bad arguments before it
touches the device."""
import ctypes
import os
import re

import pytest

import exact_tiled_attention_31_b200 as fa
from exact_tiled_attention_31_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build_library()
    return fa.load_library()


def _declared():
    names = set()
    for hdr in os.listdir(os.path.join(ROOT, "include")):
        text = open(os.path.join(ROOT, "include", hdr)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert {"fa_fwd", "fa_fwd_varlen", "fa_bwd", "fa_bwd_workspace_size"} <= names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    assert set(fa.EXPORTS) <= names


def test_status_strings(lib):
    for code in range(5):
        assert fa.fa_status_string(code).startswith("FA_")


def test_workspace_size_formula(lib):
    def up(x):
        return (x + 255) // 256 * 256
    for B, H, S, D in [(1, 32, 4096, 128), (2, 3, 17, 64), (4, 16, 8192, 128)]:
        heads, spad = B * H, (S + 127) // 128 * 128
        # two fp32 dQ accumulators, per-query rows, ordering counters (two chains), the work counter
        expect = up(2 * heads * S * D * 4) + up(heads * spad * 32) + up(heads * (spad // 128) * 2 * 4) + 256
        assert fa.fa_bwd_workspace_size(B, H, S, D) == expect
    assert fa.fa_bwd_workspace_size(1, 1, 16, 96) == 0
    assert fa.fa_bwd_workspace_size(0, 1, 16, 64) == 0


def test_fwd_argument_errors(lib):
    A = 1 << 20  # a 16-byte aligned fake address, never dereferenced
    ok = dict(q=A, k=A, v=A, o=A, lse=A, B=1, H=1, S=16, D=64, scale=0.125, causal=0, dt=0, stream=None)

    def call(**kw):
        a = {**ok, **kw}
        return fa.fa_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["S"], a["D"], a["scale"],
                         a["causal"], a["dt"], a["stream"])
    assert call(D=96) == fa.api.FA_ERR_UNSUPPORTED
    assert call(D=256) == fa.api.FA_ERR_UNSUPPORTED
    assert call(S=-1) == fa.api.FA_ERR_INVALID_ARG
    assert call(dt=7) == fa.api.FA_ERR_INVALID_ARG
    assert call(scale=0.0) == fa.api.FA_ERR_INVALID_ARG
    assert call(scale=float("nan")) == fa.api.FA_ERR_INVALID_ARG
    assert call(q=0) == fa.api.FA_ERR_INVALID_ARG
    assert call(o=A + 8) == fa.api.FA_ERR_INVALID_ARG
    assert call(B=0) == fa.api.FA_OK      # empty problem: nothing to do
    assert call(S=0, q=0) == fa.api.FA_OK


def test_varlen_and_bwd_argument_errors(lib):
    A = 1 << 20
    assert fa.fa_fwd_varlen(A, A, A, A, A, A, 2, 300, 100, 1, 64, 0.1, 1, 0, None) == fa.api.FA_ERR_INVALID_ARG
    assert fa.fa_fwd_varlen(A, A, A, A, A, A + 2, 2, 50, 100, 1, 64, 0.1, 1, 0, None) == fa.api.FA_ERR_INVALID_ARG
    assert fa.fa_fwd_varlen(A, A, A, A, A, A, 2, 50, 100, 1, 80, 0.1, 1, 0, None) == fa.api.FA_ERR_UNSUPPORTED
    assert fa.fa_fwd_varlen(A, A, A, A, A, A, 0, 50, 100, 1, 64, 0.1, 1, 0, None) == fa.api.FA_OK
    need = fa.fa_bwd_workspace_size(1, 1, 64, 64)
    args = [A] * 9 + [1, 1, 64, 64, 0.125, 1, 0, 0]
    assert fa.fa_bwd(*args, A, need - 1, None) == fa.api.FA_ERR_INVALID_ARG      # workspace too small
    assert fa.fa_bwd(*args, A + 16, need, None) == fa.api.FA_ERR_INVALID_ARG     # workspace not 256-aligned
    assert fa.fa_bwd(*([A] * 8 + [0]), 1, 1, 64, 64, 0.125, 1, 0, 0, A, need, None) == fa.api.FA_ERR_INVALID_ARG
    assert fa.fa_bwd(*([A] * 9), 1, 1, 64, 48, 0.125, 1, 0, 0, A, need, None) == fa.api.FA_ERR_UNSUPPORTED


def test_bwd_split_argument_errors(lib):
    """fa_bwd_preprocess / fa_bwd_main / fa_bwd_finish refuse bad arguments
    before launching anything (no GPU is touched here), with the same rules
    as fa_bwd; fa_bwd_finish takes the deterministic flag of fa_bwd_main."""
    A = 1 << 20
    B, H, S, D, sc, bf = 1, 2, 300, 64, 0.125, fa.api.FA_BF16
    need = fa.fa_bwd_workspace_size(B, H, S, D)
    E, U = fa.api.FA_ERR_INVALID_ARG, fa.api.FA_ERR_UNSUPPORTED
    pre = lambda ws=A, nb=need, d=D, dt=bf, o=A: fa.fa_bwd_preprocess(o, A, A, B, H, S, d, dt, ws, nb, None)
    main = lambda ws=A, nb=need, d=D, dt=bf, q=A, det=1: fa.fa_bwd_main(q, A, A, A, A, A, B, H, S, d, sc, 1, dt, det,
                                                                      ws, nb, None)
    fin = lambda ws=A, nb=need, d=D, dt=bf, dq=A, s=sc, det=1: fa.fa_bwd_finish(dq, B, H, S, d, s, dt, det, ws, nb,
                                                                               None)
    for call in (pre, main, fin):
        assert call(nb=need - 1) == E          # workspace too small
        assert call(ws=A + 16) == E            # workspace not 256-byte aligned
        assert call(ws=0) == E                 # no workspace
        assert call(d=96) == U                 # head dim not built
        assert call(dt=7) == E                 # unknown dtype
    assert pre(o=A + 2) == E                   # misaligned O
    assert main(q=0) == E                      # null Q
    assert fin(dq=A + 8) == E                  # misaligned dQ
    assert fin(s=float("nan")) == E            # bad scale
    assert fa.fa_bwd_finish(A, 0, H, S, D, sc, bf, 1, 0, 0, None) == fa.api.FA_OK   # empty batch: nothing to do


def test_missing_library_fails_loudly(tmp_path):
    saved = fa.api._lib
    fa.api._lib = None
    try:
        with pytest.raises(RuntimeError, match="missing"):
            fa.api.load_library(str(tmp_path / "nope.so"))
    finally:
        fa.api._lib = saved


def test_bwd_varlen_workspace_and_argument_errors(lib):
    def up(x):
        return (x + 255) // 256 * 256
    nseq, mx, T, H, D = 3, 300, 500, 4, 128
    spad = (mx + 127) // 128 * 128
    expect = up(2 * H * T * D * 4) + up(H * nseq * spad * 32) + up(H * nseq * (spad // 128) * 2 * 4) + 256
    assert fa.fa_bwd_varlen_workspace_size(nseq, mx, T, H, D) == expect
    assert fa.fa_bwd_varlen_workspace_size(nseq, mx, T, H, 96) == 0
    assert fa.fa_bwd_varlen_workspace_size(0, mx, T, H, D) == 0
    A = 1 << 20
    ws = fa.fa_bwd_varlen_workspace_size(2, 50, 100, 1, 64)

    def call(**kw):
        a = dict(cu=A, nseq=2, mx=50, T=100, H=1, D=64, scale=0.1, causal=1, dt=0, det=0, ws=A, wsb=ws, dq=A)
        a.update(kw)
        return fa.fa_bwd_varlen(A, A, A, A, A, A, a["dq"], A, A, a["cu"], a["nseq"], a["mx"], a["T"], a["H"], a["D"],
                                a["scale"], a["causal"], a["dt"], a["det"], a["ws"], a["wsb"], None)
    assert call(mx=300) == fa.api.FA_ERR_INVALID_ARG         # longest sequence beyond the pack
    assert call(cu=A + 2) == fa.api.FA_ERR_INVALID_ARG       # misaligned offsets
    assert call(dq=A + 8) == fa.api.FA_ERR_INVALID_ARG       # misaligned output
    assert call(ws=A + 64) == fa.api.FA_ERR_INVALID_ARG      # workspace not 256-byte aligned
    assert call(wsb=ws - 1) == fa.api.FA_ERR_INVALID_ARG     # workspace too small
    assert call(D=80) == fa.api.FA_ERR_UNSUPPORTED
    assert call(scale=-1.0) == fa.api.FA_ERR_INVALID_ARG
    assert call(nseq=0) == fa.api.FA_OK                       # empty pack: nothing to do


def test_decode_workspace_splits_and_argument_errors(lib):
    def up(x):
        return (x + 255) // 256 * 256
    for B, Hq, n, D in [(8, 32, 16, 128), (3, 5, 7, 64), (1, 1, 1, 128)]:
        assert fa.fa_decode_workspace_size(B, Hq, n, D) == up(B * Hq * n * D * 4) + up(B * Hq * n * 4)
    assert fa.fa_decode_workspace_size(1, 1, 1, 96) == 0
    assert fa.fa_decode_workspace_size(1, 1, -1, 64) == 0
    # balanced mode (n_splits = 0): one part per (cache, CTA) slot and query head,
    # at most B * Hq + 1024 CTAs x 16 heads of a group
    for B, Hq, D in [(8, 32, 128), (1, 1, 64)]:
        rows = B * Hq + 1024 * 16
        assert fa.fa_decode_workspace_size(B, Hq, 0, D) == up(rows * D * 4) + up(rows * 4)
    # the library's split choice: 1..64, at least 256 keys per split
    for B, Hkv, L in [(8, 8, 8192), (1, 1, 100), (1, 8, 32768), (64, 8, 2048), (1, 1, 1 << 20)]:
        n = fa.fa_decode_num_splits(B, Hkv, L)
        assert 1 <= n <= 64 and (n == 1 or L >= 256 * n)
    assert fa.fa_decode_num_splits(0, 8, 1024) == 1
    A = 1 << 20
    ws = fa.fa_decode_workspace_size(2, 8, 4, 64)

    def call(**kw):
        a = dict(q=A, lens=A, B=2, Hq=8, Hkv=2, L=100, D=64, scale=0.125, dt=0, n=4, ws=A, wsb=ws)
        a.update(kw)
        return fa.fa_decode(a["q"], A, A, a["lens"], A, A, a["B"], a["Hq"], a["Hkv"], a["L"], a["D"], a["scale"],
                            a["dt"], a["n"], a["ws"], a["wsb"], None)
    assert call(Hkv=3) == fa.api.FA_ERR_INVALID_ARG            # Hq not a multiple of Hkv
    assert call(Hkv=0) == fa.api.FA_ERR_INVALID_ARG
    assert call(Hq=34, Hkv=2, wsb=1 << 30) == fa.api.FA_ERR_UNSUPPORTED   # group of 17 query heads
    assert call(D=96) == fa.api.FA_ERR_UNSUPPORTED
    assert call(n=-1) == fa.api.FA_ERR_INVALID_ARG
    assert call(n=1025) == fa.api.FA_ERR_INVALID_ARG
    assert call(n=0, wsb=fa.fa_decode_workspace_size(2, 8, 0, 64) - 1) == fa.api.FA_ERR_INVALID_ARG
    assert call(lens=A + 2) == fa.api.FA_ERR_INVALID_ARG      # misaligned seq_lens
    assert call(q=A + 8) == fa.api.FA_ERR_INVALID_ARG         # misaligned q
    assert call(ws=A + 64) == fa.api.FA_ERR_INVALID_ARG       # workspace not 256-byte aligned
    assert call(wsb=ws - 1) == fa.api.FA_ERR_INVALID_ARG      # workspace too small
    assert call(scale=0.0) == fa.api.FA_ERR_INVALID_ARG
    assert call(dt=5) == fa.api.FA_ERR_INVALID_ARG
    assert call(L=-1) == fa.api.FA_ERR_INVALID_ARG
    assert call(B=0) == fa.api.FA_OK                          # empty batch: nothing to do


def test_dropout_argument_errors(lib):
    A = 1 << 20
    fwd = dict(q=A, k=A, v=A, o=A, lse=A, B=1, H=1, S=16, D=64, scale=0.125, causal=0, dt=0, p=0.1, seed=1,
               off=0, stream=None)

    def f(**kw):
        a = {**fwd, **kw}
        return fa.fa_fwd_dropout(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["S"], a["D"],
                                 a["scale"], a["causal"], a["dt"], a["p"], a["seed"], a["off"], a["stream"])
    assert f(p=-0.1) == fa.api.FA_ERR_INVALID_ARG
    assert f(p=1.0) == fa.api.FA_ERR_INVALID_ARG
    assert f(p=float("nan")) == fa.api.FA_ERR_INVALID_ARG
    assert f(D=96) == fa.api.FA_ERR_UNSUPPORTED
    assert f(o=A + 8) == fa.api.FA_ERR_INVALID_ARG
    assert f(B=0) == fa.api.FA_OK
    assert f(seed=(1 << 64) - 1, B=0) == fa.api.FA_OK          # any 64-bit seed and offset
    need = fa.fa_bwd_workspace_size(1, 1, 64, 64)

    def b(p=0.1, wsb=need, ws=A, D=64):
        return fa.fa_bwd_dropout(*([A] * 9), 1, 1, 64, D, 0.125, 1, 0, 0, p, 7, 3, ws, wsb, None)
    assert b(p=1.5) == fa.api.FA_ERR_INVALID_ARG
    assert b(wsb=need - 1) == fa.api.FA_ERR_INVALID_ARG
    assert b(ws=A + 16) == fa.api.FA_ERR_INVALID_ARG
    assert b(D=48) == fa.api.FA_ERR_UNSUPPORTED


def test_decode_split_rule():
    """The library's split count: the fewest splits giving about 0.8 x 148
    CTAs (one B200 wave), at least 256 keys each, at most 64 (148 SMs is the
    count the library assumes when no device answers)."""
    import math
    for B, Hkv, L in [(8, 8, 8192), (1, 8, 32768), (32, 8, 2048), (8, 32, 4096), (16, 1, 8192), (64, 8, 1024),
                      (1, 1, 1 << 20), (2, 4, 300)]:
        target = (8 * 148 + 9) // 10
        nmax = max(1, min(64, ((L + 31) // 32) // 8))
        expect = max(1, min(nmax, math.ceil(target / (B * Hkv))))
        assert fa.fa_decode_num_splits(B, Hkv, L) == expect, (B, Hkv, L)
