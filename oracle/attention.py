"""Plain, slow, fp64 CPU oracle for exact scaled dot-product attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
this module.  It shares no code with the CUDA path and imports nothing from
the ``exact_tiled_attention_31_b200`` package.

What it computes and where the pages define it
----------------------------------------------
The method on the pages is *exact* attention: apart from floating-point
summation order, the tiled kernel returns the plain result
``O = softmax(Q K^T * scale [+ causal mask]) V`` ("Flash Attention 的算法设计原理"
(algomooc), "FlashAttention 的定位"; "From Self-Attention to FlashAttention"
(wmrh.cn), §二 says the online result is numerically equivalent, not an
approximation).  So the oracle is that definition written out:

* scores ``s_ij = scale * q_i . k_j`` materialised in full
  ("ops-transformer里的FlashAttention" (mhpn.cn), "FlashAttention的核心思路",
  step 1 of the conventional flow);
* the three-pass stable softmax - max, then sum of exponentials, then divide
  ("From Self-Attention to FlashAttention", §二, first paragraph);
* ``O = P V`` (same conventional flow, step 3);
* the per-row log-sum-exp ``LSE_i = m_i + ln l_i`` (natural log of the sum of
  exponentials of the scaled scores) - the "statistics" the forward keeps so
  that the backward can rebuild the local blocks ("Flash Attention 的算法设计原理",
  "核心机制", third item).

The causal mask lets query ``i`` see keys ``j <= i`` (diagonal included,
top-left aligned; "ops-transformer里的FlashAttention", "实战踩坑 坑二").  In a
packed variable-length batch each sequence only sees itself, and causality is
counted from the sequence's own start.

The pages give no backward formulas (only that it recomputes local blocks
from saved statistics), so the gradients are the textbook ones for
``L = sum(dO * O)``::

    dV_j  = sum_i P_ij dO_i
    dP_ij = dO_i . v_j
    D_i   = sum_j P_ij dP_ij            (= dO_i . O_i)
    dS_ij = P_ij (dP_ij - D_i)
    dQ_i  = scale * sum_j dS_ij k_j
    dK_j  = scale * sum_i dS_ij q_i

Readings where the pages are silent: a row with no visible key (cannot occur
with equal query/key lengths) returns ``O = 0`` and ``LSE = -inf``.  Large
inputs are processed a block of query rows at a time; every row still goes
through its own full three passes, so only memory use changes.

``attention_forward_online`` restates the one-pass running-max / running-sum
update of "From Self-Attention to FlashAttention", §二 (unnormalised output
rescaled by ``exp(m_prev - m_new)``, divided once at the end).  It exists
only so the tests can check that the one-pass form equals the three-pass
one; the printed update in "ops-transformer里的FlashAttention", "在线softmax",
divides by the running sum inside the loop and is not used.

All inputs are converted to float64 exactly (bf16/fp16 values are exactly
representable) before any arithmetic.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "to_f64",
    "attention_scores",
    "attention_probs",
    "attention_forward",
    "attention_forward_rows",
    "attention_backward",
    "attention_forward_online",
    "varlen_forward",
    "varlen_backward",
    "decode_forward",
    "merge_partials",
    "philox4x32_10",
    "dropout_keep_threshold",
    "dropout_scale",
    "dropout_keep",
    "attention_forward_dropout",
    "attention_backward_dropout",
    "varlen_forward_dropout",
    "varlen_backward_dropout",
    "flop_count",
]

_ROW_BLOCK = 1024


def to_f64(x) -> np.ndarray:
    """Exact conversion of a torch tensor / array of bf16, fp16 or fp32 to float64."""
    if hasattr(x, "detach"):  # torch tensor, without importing torch here
        x = x.detach().cpu()
        if str(x.dtype) in ("torch.bfloat16", "torch.float16"):
            x = x.float()  # exact widening; numpy has no bfloat16
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def _visible(nq: int, nk: int, causal: bool, q_rows: np.ndarray | None = None) -> np.ndarray:
    """Boolean [nq, nk] mask of the keys each query row may attend to."""
    rows = np.arange(nq) if q_rows is None else np.asarray(q_rows)
    cols = np.arange(nk)
    if causal:
        return cols[None, :] <= rows[:, None]
    return np.ones((rows.shape[0], nk), dtype=bool)


def attention_scores(q: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """s = scale * q k^T for one head: q [Sq, D], k [Sk, D] -> [Sq, Sk]."""
    return scale * (q @ k.T)


def _three_pass(s: np.ndarray, vis: np.ndarray):
    """Stable softmax of each row over its visible keys, in three passes.

    Returns (P, m, l) with P [rows, keys], m the row maximum and l the sum of
    exp(s - m) over the visible keys.
    """
    masked = np.where(vis, s, -np.inf)
    m = masked.max(axis=1)                                  # pass 1: maximum
    m_safe = np.where(np.isfinite(m), m, 0.0)
    e = np.where(vis, np.exp(masked - m_safe[:, None]), 0.0)
    l = e.sum(axis=1)                                        # pass 2: sum of exp
    with np.errstate(invalid="ignore", divide="ignore"):
        p = np.where(l[:, None] > 0, e / l[:, None], 0.0)     # pass 3: divide
    return p, m, l


def attention_probs(q, k, scale: float, causal: bool) -> np.ndarray:
    """Full probability matrix P for one head (small inputs only)."""
    q, k = to_f64(q), to_f64(k)
    s = attention_scores(q, k, scale)
    p, _, _ = _three_pass(s, _visible(q.shape[0], k.shape[0], causal))
    return p


def _head_forward(q, k, v, scale, causal, rows=None):
    nq = q.shape[0] if rows is None else len(rows)
    row_ids = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    o = np.zeros((nq, v.shape[1]))
    lse = np.empty(nq)
    for b0 in range(0, nq, _ROW_BLOCK):
        r = row_ids[b0:b0 + _ROW_BLOCK]
        s = attention_scores(q[r], k, scale)
        p, m, l = _three_pass(s, _visible(q.shape[0], k.shape[0], causal, r))
        o[b0:b0 + len(r)] = p @ v
        with np.errstate(divide="ignore"):
            lse[b0:b0 + len(r)] = np.where(l > 0, m + np.log(l), -np.inf)
    return o, lse


def attention_forward(q, k, v, scale: float, causal: bool, heads=None):
    """O and LSE for [B, H, S, D] inputs (or [S, D] for a single head).

    ``heads`` optionally restricts the work to a list of (b, h) pairs; the
    result then has shape [len(heads), S, D] / [len(heads), S].
    """
    q, k, v = to_f64(q), to_f64(k), to_f64(v)
    if q.ndim == 2:
        return _head_forward(q, k, v, scale, causal)
    B, H, S, D = q.shape
    pairs = [(b, h) for b in range(B) for h in range(H)] if heads is None else list(heads)
    o = np.zeros((len(pairs), S, v.shape[-1]))
    lse = np.zeros((len(pairs), S))
    for n, (b, h) in enumerate(pairs):
        o[n], lse[n] = _head_forward(q[b, h], k[b, h], v[b, h], scale, causal)
    if heads is None:
        return o.reshape(B, H, S, -1), lse.reshape(B, H, S)
    return o, lse


def attention_forward_rows(q, k, v, scale: float, causal: bool, b: int, h: int, rows):
    """O and LSE of selected query rows of head (b, h) - for full-size spot checks."""
    q, k, v = to_f64(q[b, h]), to_f64(k[b, h]), to_f64(v[b, h])
    return _head_forward(q, k, v, scale, causal, rows=np.asarray(rows))


def _head_backward(q, k, v, do, scale, causal):
    s = attention_scores(q, k, scale)
    p, _, _ = _three_pass(s, _visible(q.shape[0], k.shape[0], causal))
    o = p @ v
    dv = p.T @ do
    dp = do @ v.T
    d_row = (p * dp).sum(axis=1)
    ds = p * (dp - d_row[:, None])
    dq = scale * (ds @ k)
    dk = scale * (ds.T @ q)
    return dq, dk, dv, o


def attention_backward(q, k, v, do, scale: float, causal: bool, heads=None):
    """dQ, dK, dV of L = sum(dO * O) for [B, H, S, D] (or [S, D]) inputs."""
    q, k, v, do = to_f64(q), to_f64(k), to_f64(v), to_f64(do)
    if q.ndim == 2:
        return _head_backward(q, k, v, do, scale, causal)[:3]
    B, H, S, D = q.shape
    pairs = [(b, h) for b in range(B) for h in range(H)] if heads is None else list(heads)
    dq = np.zeros((len(pairs), S, D))
    dk = np.zeros((len(pairs), S, D))
    dv = np.zeros((len(pairs), S, v.shape[-1]))
    for n, (b, h) in enumerate(pairs):
        dq[n], dk[n], dv[n], _ = _head_backward(q[b, h], k[b, h], v[b, h], do[b, h], scale, causal)
    if heads is None:
        return dq.reshape(q.shape), dk.reshape(k.shape), dv.reshape(v.shape)
    return dq, dk, dv


def attention_forward_online(q, k, v, scale: float, causal: bool, block: int = 128):
    """One-pass online-softmax attention for one head, [S, D] inputs.

    Key/value blocks of ``block`` rows are visited once; for each, every query
    row updates its running max, rescales its running sum and unnormalised
    output by exp(m_prev - m_new), and adds the block's contribution; the
    output is divided by the running sum at the end.
    """
    q, k, v = to_f64(q), to_f64(k), to_f64(v)
    nq, nk = q.shape[0], k.shape[0]
    o = np.zeros((nq, v.shape[1]))
    m = np.full(nq, -np.inf)
    l = np.zeros(nq)
    for j0 in range(0, nk, block):
        kj, vj = k[j0:j0 + block], v[j0:j0 + block]
        s = attention_scores(q, kj, scale)
        if causal:
            cols = np.arange(j0, j0 + kj.shape[0])
            s = np.where(cols[None, :] <= np.arange(nq)[:, None], s, -np.inf)
        m_new = np.maximum(m, s.max(axis=1))
        m_ref = np.where(np.isfinite(m_new), m_new, 0.0)
        corr = np.exp(np.where(np.isfinite(m), m - m_ref, -np.inf))
        p = np.exp(s - m_ref[:, None])
        l = corr * l + p.sum(axis=1)
        o = corr[:, None] * o + p @ vj
        m = m_new
    with np.errstate(invalid="ignore", divide="ignore"):
        out = np.where(l[:, None] > 0, o / l[:, None], 0.0)
        lse = np.where(l > 0, m + np.log(l), -np.inf)
    return out, lse


def _seq_bounds(cu_seqlens):
    cu = [int(x) for x in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    return list(zip(cu[:-1], cu[1:]))


def varlen_forward(q, k, v, cu_seqlens, scale: float, causal: bool, heads=None, seqs=None):
    """Packed [H, T, D] forward: each sequence attends only within itself.

    Returns O [H', T, D] and LSE [H', T] for the heads in ``heads`` (all by
    default); rows of sequences not in ``seqs`` are left at zero.
    """
    q, k, v = to_f64(q), to_f64(k), to_f64(v)
    H, T, D = q.shape
    heads = list(range(H)) if heads is None else list(heads)
    bounds = _seq_bounds(cu_seqlens)
    seqs = range(len(bounds)) if seqs is None else seqs
    o = np.zeros((len(heads), T, v.shape[-1]))
    lse = np.zeros((len(heads), T))
    for n, h in enumerate(heads):
        for si in seqs:
            a, b = bounds[si]
            o[n, a:b], lse[n, a:b] = _head_forward(q[h, a:b], k[h, a:b], v[h, a:b], scale, causal)
    return o, lse


def varlen_backward(q, k, v, do, cu_seqlens, scale: float, causal: bool, heads=None):
    """Packed [H, T, D] gradients, one sequence at a time."""
    q, k, v, do = to_f64(q), to_f64(k), to_f64(v), to_f64(do)
    H, T, D = q.shape
    heads = list(range(H)) if heads is None else list(heads)
    dq = np.zeros((len(heads), T, D))
    dk = np.zeros((len(heads), T, D))
    dv = np.zeros((len(heads), T, v.shape[-1]))
    for n, h in enumerate(heads):
        for a, b in _seq_bounds(cu_seqlens):
            dq[n, a:b], dk[n, a:b], dv[n, a:b], _ = _head_backward(
                q[h, a:b], k[h, a:b], v[h, a:b], do[h, a:b], scale, causal)
    return dq, dk, dv


def decode_forward(q, k_cache, v_cache, seq_lens, scale: float):
    """One new query token per (sequence, query head) against its KV cache.

    ``q`` [B, Hq, D]; ``k_cache``, ``v_cache`` [B, Hkv, L, D] with Hq a
    multiple of Hkv: query head h reads KV head ``h // (Hq // Hkv)``
    (grouped-query attention; Hkv = Hq is multi-head, Hkv = 1 multi-query).
    Sequence b holds ``seq_lens[b]`` valid cached keys.  The new token is the
    last position, so every cached key is visible and each (b, h) is the plain
    definition for a single query row.  Returns O [B, Hq, D] and LSE [B, Hq].
    Decode reads the KV cache once per generated token, with GQA/MQA sharing
    one KV head among several query heads ("Flash Attention 的算法设计原理",
    "训练与推理价值" and "练习口述回答").
    """
    q, k, v = to_f64(q), to_f64(k_cache), to_f64(v_cache)
    B, Hq, D = q.shape
    Hkv = k.shape[1]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    group = Hq // Hkv
    lens = [int(x) for x in (seq_lens.tolist() if hasattr(seq_lens, "tolist") else seq_lens)]
    o = np.zeros((B, Hq, v.shape[-1]))
    lse = np.zeros((B, Hq))
    for b in range(B):
        L = lens[b]
        for h in range(Hq):
            kv = h // group
            ob, lb = _head_forward(q[b, h][None, :], k[b, kv, :L], v[b, kv, :L], scale, False)
            o[b, h], lse[b, h] = ob[0], lb[0]
    return o, lse


def merge_partials(o_parts, lse_parts):
    """Combine results of the same query rows over disjoint key subsets.

    ``o_parts`` [S, ..., D] (each normalised over its own subset) and
    ``lse_parts`` [S, ...]: since exp(LSE_s) is the subset's sum of
    exponentials, LSE = log sum_s exp(LSE_s) and O = sum_s exp(LSE_s - LSE) O_s
    (the same rescaling as the running update of "From Self-Attention to
    FlashAttention", §二, applied once per subset).  Subsets with no key carry
    LSE = -inf and weight 0.
    """
    o_parts, lse_parts = to_f64(o_parts), to_f64(lse_parts)
    m = lse_parts.max(axis=0)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(lse_parts - m_safe)
    tot = w.sum(axis=0)
    with np.errstate(divide="ignore", invalid="ignore"):
        lse = np.where(tot > 0, m_safe + np.log(tot), -np.inf)
        o = np.where(tot[..., None] > 0, (w[..., None] * o_parts).sum(axis=0) / tot[..., None], 0.0)
    return o, lse


# ---------------------------------------------------------------- dropout
#
# Dropout on the attention probabilities, the branch the pages ask to be
# tested on its own ("Flash Attention 的算法设计原理", "练习口述回答": dropout is
# one of the paths to cover separately; the mask has to be regenerated in the
# backward rather than stored, which needs a counter-based generator).  The
# pages fix neither the generator nor where the mask sits, so the reading is:
#
# * P is the exact softmax; the output uses  Pd = P * M * s  with M_ij in
#   {0, 1} (kept with probability t / 2^8, t below) and s = 2^8 / t;
#   O = Pd V.  LSE is the statistic of the undropped softmax (dropout comes
#   after normalisation).
# * M_ij for head bh (= b * H + h), query i, key j is decided by one byte of
#   one Philox4x32-10 output (Salmon, Moraes, Dror and Shaw, "Parallel random
#   numbers: as easy as 1, 2, 3", SC 2011) with
#       counter = (j >> 3, i >> 1, bh, offset mod 2^32),
#       key     = (seed mod 2^32, seed >> 32 mod 2^32):
#   word number 2 * (i & 1) + ((j >> 2) & 1), byte j & 3 of it (the lowest
#   for j & 3 = 0).  The element is kept when that byte is below
#   t = floor((1 - p) * 2^8) (t >= 1), so an element is kept with
#   probability t / 2^8 exactly (p is taken to the next multiple of 2^-8
#   above it, or equal), and kept values are scaled by 2^8 / t, which keeps
#   E[O] = O exactly.  One call covers a 2 x 8 (query, key) block.
# * Backward of L = sum(dO * O) with the same M:
#       dV = Pd^T dO,  dPd = dO V^T,  dP = dPd * M * s,
#       D_i = sum_j P_ij dP_ij  (= dO_i . O_i),  dS = P * (dP - D),
#       dQ = scale dS K,  dK = scale dS^T Q.

_MASK32 = np.uint64(0xFFFFFFFF)
_PHILOX_M = (np.uint64(0xD2511F53), np.uint64(0xCD9E8D57))   # round multipliers
_PHILOX_W = (np.uint64(0x9E3779B9), np.uint64(0xBB67AE85))   # key schedule increments


def philox4x32_10(ctr, key):
    """Philox4x32 with 10 rounds on broadcastable uint32 counter words.

    ``ctr`` is four arrays (c0, c1, c2, c3), ``key`` two integers (k0, k1).
    Each round multiplies c0 and c2 by the two round constants, keeps the
    64-bit products' halves, and mixes them with c1, c3 and the round key:
    (c0, c1, c2, c3) <- (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1,
    lo(M0 c0)); the key advances by the Weyl increments between rounds.
    Returns the four output words as uint32 arrays.
    """
    c = [np.asarray(x).astype(np.uint64) & _MASK32 for x in ctr]
    c = np.broadcast_arrays(*c)
    k0, k1 = np.uint64(int(key[0]) & 0xFFFFFFFF), np.uint64(int(key[1]) & 0xFFFFFFFF)
    for r in range(10):
        if r:
            k0 = (k0 + _PHILOX_W[0]) & _MASK32
            k1 = (k1 + _PHILOX_W[1]) & _MASK32
        p0 = c[0] * _PHILOX_M[0]   # < 2^64: exact in uint64
        p1 = c[2] * _PHILOX_M[1]
        c = [(p1 >> np.uint64(32)) ^ c[1] ^ k0, p1 & _MASK32, (p0 >> np.uint64(32)) ^ c[3] ^ k1, p0 & _MASK32]
    return [x.astype(np.uint32) for x in c]


def dropout_keep_threshold(p: float) -> int:
    """8-bit threshold t = max(1, floor((1 - p) 2^8)): a byte below it keeps the element."""
    if not 0.0 <= p < 1.0:
        raise ValueError("dropout probability must be in [0, 1)")
    return max(1, int(np.floor((1.0 - p) * 256.0)))


def dropout_scale(p: float) -> float:
    """Scale of the kept values, 2^8 / t (1 / the exact keep probability); 1 for p = 0."""
    return 256.0 / dropout_keep_threshold(p)


def dropout_keep(bh: int, rows, cols, p: float, seed: int, offset: int) -> np.ndarray:
    """Boolean keep mask [len(rows), len(cols)] of head bh (query rows, key columns).

    Element (i, j) reads byte (j & 3) of word 2 (i & 1) + ((j >> 2) & 1) of
    Philox4x32-10 at counter (j >> 3, i >> 1, bh, offset), key (seed low,
    seed high 32 bits): one call covers a 2 x 8 (query, key) block.
    """
    i = np.asarray(rows, dtype=np.int64)[:, None]
    j = np.asarray(cols, dtype=np.int64)[None, :]
    words = philox4x32_10((j >> 3, i >> 1, bh, offset & 0xFFFFFFFF), (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF))
    sel = 2 * (i & 1) + ((j >> 2) & 1)
    w = np.choose(np.broadcast_to(sel, np.broadcast_shapes(i.shape, j.shape)), words).astype(np.int64)
    byte = (w >> (8 * (j & 3))) & 0xFF
    return byte < dropout_keep_threshold(p)


def _head_dropout(q, k, v, do, scale, causal, p, keep):
    s = attention_scores(q, k, scale)
    pr, m, l = _three_pass(s, _visible(q.shape[0], k.shape[0], causal))
    pd = pr * keep * dropout_scale(p)
    o = pd @ v
    with np.errstate(divide="ignore"):
        lse = np.where(l > 0, m + np.log(l), -np.inf)
    if do is None:
        return o, lse
    dv = pd.T @ do
    dp = (do @ v.T) * keep * dropout_scale(p)
    d_row = (pr * dp).sum(axis=1)
    ds = pr * (dp - d_row[:, None])
    return scale * (ds @ k), scale * (ds.T @ q), dv


def attention_forward_dropout(q, k, v, scale: float, causal: bool, p: float, seed: int, offset: int, heads=None):
    """O, LSE with dropout on P for [B, H, S, D] inputs (LSE of the undropped softmax)."""
    q, k, v = to_f64(q), to_f64(k), to_f64(v)
    B, H, S, D = q.shape
    pairs = [(b, h) for b in range(B) for h in range(H)] if heads is None else list(heads)
    o = np.zeros((len(pairs), S, v.shape[-1]))
    lse = np.zeros((len(pairs), S))
    for n, (b, h) in enumerate(pairs):
        keep = dropout_keep(b * H + h, np.arange(S), np.arange(S), p, seed, offset)
        o[n], lse[n] = _head_dropout(q[b, h], k[b, h], v[b, h], None, scale, causal, p, keep)
    if heads is None:
        return o.reshape(B, H, S, -1), lse.reshape(B, H, S)
    return o, lse


def attention_backward_dropout(q, k, v, do, scale: float, causal: bool, p: float, seed: int, offset: int,
                               heads=None):
    """dQ, dK, dV of L = sum(dO * O) with the dropout mask of the forward."""
    q, k, v, do = to_f64(q), to_f64(k), to_f64(v), to_f64(do)
    B, H, S, D = q.shape
    pairs = [(b, h) for b in range(B) for h in range(H)] if heads is None else list(heads)
    out = [np.zeros((len(pairs), S, D)) for _ in range(2)] + [np.zeros((len(pairs), S, v.shape[-1]))]
    for n, (b, h) in enumerate(pairs):
        keep = dropout_keep(b * H + h, np.arange(S), np.arange(S), p, seed, offset)
        g = _head_dropout(q[b, h], k[b, h], v[b, h], do[b, h], scale, causal, p, keep)
        for t, x in zip(out, g):
            t[n] = x
    if heads is None:
        return tuple(t.reshape(B, H, S, -1) for t in out)
    return tuple(out)


def varlen_forward_dropout(q, k, v, cu_seqlens, scale: float, causal: bool, p: float, seed: int, offset: int,
                           heads=None):
    """Packed [H, T, D] forward with dropout on P.

    Reading (the pages give no packed layout for the mask): sequence s of the
    pack takes the mask a dense batch would give its batch index s, i.e.
    head index s * H + h, query and key indices counted from the sequence's
    own first token.  A pack of equal lengths therefore drops exactly what
    the dense [nseq, H, L, D] batch drops.
    """
    q, k, v = to_f64(q), to_f64(k), to_f64(v)
    H, T, D = q.shape
    heads = list(range(H)) if heads is None else list(heads)
    o = np.zeros((len(heads), T, v.shape[-1]))
    lse = np.zeros((len(heads), T))
    for n, h in enumerate(heads):
        for si, (a, b) in enumerate(_seq_bounds(cu_seqlens)):
            L = b - a
            keep = dropout_keep(si * H + h, np.arange(L), np.arange(L), p, seed, offset)
            o[n, a:b], lse[n, a:b] = _head_dropout(q[h, a:b], k[h, a:b], v[h, a:b], None, scale, causal, p, keep)
    return o, lse


def varlen_backward_dropout(q, k, v, do, cu_seqlens, scale: float, causal: bool, p: float, seed: int, offset: int,
                            heads=None):
    """dQ, dK, dV of a packed [H, T, D] batch with the mask of varlen_forward_dropout."""
    q, k, v, do = to_f64(q), to_f64(k), to_f64(v), to_f64(do)
    H, T, D = q.shape
    heads = list(range(H)) if heads is None else list(heads)
    out = [np.zeros((len(heads), T, D)) for _ in range(2)] + [np.zeros((len(heads), T, v.shape[-1]))]
    for n, h in enumerate(heads):
        for si, (a, b) in enumerate(_seq_bounds(cu_seqlens)):
            L = b - a
            keep = dropout_keep(si * H + h, np.arange(L), np.arange(L), p, seed, offset)
            g = _head_dropout(q[h, a:b], k[h, a:b], v[h, a:b], do[h, a:b], scale, causal, p, keep)
            for t, x in zip(out, g):
                t[n, a:b] = x
    return tuple(out)


def flop_count(lengths, heads: int, d: int, causal: bool) -> tuple[float, float]:
    """(forward, backward) FLOPs by the usual convention.

    Forward counts the two matrix products, 4 * S^2 * D per head, halved
    under a causal mask; backward counts five products, 2.5x the forward.
    """
    f = sum(4.0 * L * L * d for L in lengths) * heads
    if causal:
        f *= 0.5
    return f, 2.5 * f
