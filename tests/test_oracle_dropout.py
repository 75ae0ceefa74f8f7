"""CPU pins of the oracle's dropout branch: the counter-based generator's
statistics, the keep rate, determinism in (seed, offset, head), the p = 0
reduction to plain attention, unbiasedness of the dropped output, and the
backward against central finite differences for a fixed mask.  Planted
mistakes (a missing 1/(1-p), the mask applied to P inside dS, a mask that
ignores the head) each fail one of them."""
import json
import math
import os

import numpy as np
import pytest

from oracle import attention as oa

_KAT = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.json")


def _kat_vectors():
    with open(_KAT) as f:
        vecs = json.load(f)["vectors"]
    return [([int(x, 16) for x in v["ctr"]], [int(x, 16) for x in v["key"]], [int(x, 16) for x in v["out"]])
            for v in vecs]


def _kat_failures(gen):
    """Known-answer vectors that ``gen`` does not reproduce."""
    bad = []
    for ctr, key, out in _kat_vectors():
        got = [int(np.asarray(w)) for w in gen(ctr, key)]
        if got != out:
            bad.append((ctr, key, [hex(x) for x in got]))
    return bad


def test_philox_known_answers():
    """The oracle's generator reproduces the published Philox4x32-10
    known-answer vectors (Salmon, Moraes, Dror and Shaw, SC 2011; the
    Random123 distribution's kat_vectors): the all-zero, all-ones and
    pi-digit counters and keys, stored in tests/golden/philox4x32_10_kat.json.
    This pins the generator to its published definition, independently of
    the GPU copy agreeing with it."""
    assert _kat_failures(oa.philox4x32_10) == []


def test_philox_known_answers_reject_planted_mistakes(monkeypatch):
    """Each plausible slip in a Philox implementation fails the known
    answers: the two round multipliers swapped, a wrong Weyl increment, nine
    rounds instead of ten (key schedule one step short), and output words
    in the wrong order."""
    m0, m1 = oa._PHILOX_M
    w0, w1 = oa._PHILOX_W
    with monkeypatch.context() as mp:
        mp.setattr(oa, "_PHILOX_M", (m1, m0))
        assert len(_kat_failures(oa.philox4x32_10)) == 3
    with monkeypatch.context() as mp:
        mp.setattr(oa, "_PHILOX_W", (w0, np.uint64(0xBB67AE86)))
        assert len(_kat_failures(oa.philox4x32_10)) == 3
    with monkeypatch.context() as mp:
        mp.setattr(oa, "_PHILOX_W", (w1, w0))
        assert len(_kat_failures(oa.philox4x32_10)) == 3

    def nine_rounds(ctr, key):
        c = [np.asarray(x).astype(np.uint64) for x in ctr]
        k0, k1 = np.uint64(key[0]), np.uint64(key[1])
        mask = np.uint64(0xFFFFFFFF)
        for r in range(9):
            if r:
                k0, k1 = (k0 + w0) & mask, (k1 + w1) & mask
            p0, p1 = c[0] * m0, c[2] * m1
            c = [(p1 >> np.uint64(32)) ^ c[1] ^ k0, p1 & mask, (p0 >> np.uint64(32)) ^ c[3] ^ k1, p0 & mask]
        return c

    assert len(_kat_failures(nine_rounds)) == 3

    def swapped_words(ctr, key):
        x = oa.philox4x32_10(ctr, key)
        return [x[1], x[0], x[2], x[3]]

    assert len(_kat_failures(swapped_words)) == 3


def _qkv(S, D, seed, B=1, H=1):
    g = np.random.default_rng(seed)
    return [g.standard_normal((B, H, S, D)) for _ in range(4)]


def test_philox_output_statistics():
    """2^18 words from 2^16 counters: every bit set about half the time, top
    byte uniform (chi-square), no repeated 128-bit block, and one flipped
    counter bit changes about half of the 128 output bits."""
    c0 = np.arange(1 << 16, dtype=np.int64)
    words = np.stack(oa.philox4x32_10((c0, 17, 3, 0), (0x12345678, 0x9ABCDEF0)), axis=1)  # [N, 4]
    flat = words.reshape(-1).astype(np.uint64)
    n = flat.size
    for bit in range(32):
        ones = int(((flat >> np.uint64(bit)) & np.uint64(1)).sum())
        assert abs(ones - n / 2) < 5 * math.sqrt(n / 4), f"bit {bit}: {ones} of {n}"
    top = (flat >> np.uint64(24)).astype(np.int64)
    hist = np.bincount(top, minlength=256)
    chi2 = ((hist - n / 256) ** 2 / (n / 256)).sum()
    assert chi2 < 255 + 6 * math.sqrt(2 * 255), chi2
    assert len({tuple(r) for r in words.tolist()}) == words.shape[0]
    base = np.stack(oa.philox4x32_10((c0[:4096], 5, 6, 7), (1, 2)), axis=1).astype(np.uint64)
    flips = []
    for word in range(4):
        for bit in (0, 7, 19, 31):
            ctr = [c0[:4096], np.full(4096, 5), np.full(4096, 6), np.full(4096, 7)]
            ctr[word] = ctr[word] ^ (1 << bit)
            out = np.stack(oa.philox4x32_10(ctr, (1, 2)), axis=1).astype(np.uint64)
            diff = out ^ base
            flips.append(sum(int(bin(int(x)).count("1")) for x in diff[:256].reshape(-1)) / 256)
    assert all(56 < f < 72 for f in flips), flips


@pytest.mark.parametrize("p", [0.1, 0.5, 0.9])
def test_keep_rate(p):
    keep = oa.dropout_keep(5, np.arange(512), np.arange(512), p, seed=99, offset=3)
    n = keep.size
    q = oa.dropout_keep_threshold(p) / 256.0  # exact keep probability, within 2^-8 of 1 - p
    assert abs(q - (1 - p)) <= 2.0 ** -8
    assert abs(keep.mean() - q) < 5 * math.sqrt(q * (1 - q) / n)
    assert oa.dropout_scale(p) == 1.0 / q


def test_mask_is_a_function_of_seed_offset_and_head():
    a = oa.dropout_keep(2, np.arange(64), np.arange(64), 0.5, seed=7, offset=1)
    assert np.array_equal(a, oa.dropout_keep(2, np.arange(64), np.arange(64), 0.5, seed=7, offset=1))
    for other in (dict(bh=3, seed=7, offset=1), dict(bh=2, seed=8, offset=1), dict(bh=2, seed=7, offset=2),
                  dict(bh=2, seed=7 + (1 << 32), offset=1)):
        b = oa.dropout_keep(other["bh"], np.arange(64), np.arange(64), 0.5, seed=other["seed"], offset=other["offset"])
        agree = (a == b).mean()
        assert 0.4 < agree < 0.6, (other, agree)  # independent masks agree on about half
    # a sub-block of rows and columns is the same as the corresponding slice
    sub = oa.dropout_keep(2, np.arange(10, 30), np.arange(33, 61), 0.5, seed=7, offset=1)
    assert np.array_equal(sub, a[10:30, 33:61])


def test_p_zero_is_plain_attention():
    q, k, v, do = _qkv(40, 16, seed=1, B=2, H=2)
    for causal in (False, True):
        o, lse = oa.attention_forward_dropout(q, k, v, 0.3, causal, 0.0, seed=1, offset=0)
        o0, lse0 = oa.attention_forward(q, k, v, 0.3, causal)
        assert np.array_equal(o, o0) and np.array_equal(lse, lse0)
        g = oa.attention_backward_dropout(q, k, v, do, 0.3, causal, 0.0, seed=1, offset=0)
        g0 = oa.attention_backward(q, k, v, do, 0.3, causal)
        for a, b in zip(g, g0):
            assert np.allclose(a, b, rtol=0, atol=1e-13)


def test_lse_is_that_of_the_undropped_softmax():
    q, k, v, _ = _qkv(50, 8, seed=2, H=3)
    _, lse = oa.attention_forward_dropout(q, k, v, 0.4, True, 0.3, seed=11, offset=5)
    _, lse0 = oa.attention_forward(q, k, v, 0.4, True)
    assert np.array_equal(lse, lse0)


def _mean_over_offsets(fwd, q, k, v, p, n):
    acc = np.zeros(q.shape[:-1] + (v.shape[-1],))
    sq = np.zeros_like(acc)
    for off in range(n):
        o, _ = fwd(q, k, v, 0.5, False, p, seed=21, offset=off)
        acc += o
        sq += o * o
    mean = acc / n
    std = np.sqrt(np.maximum(sq / n - mean * mean, 0.0))
    return mean, std


def test_dropped_output_is_unbiased():
    """E[O_drop] = O: the mean over 400 independent masks stays within five
    standard errors of the plain output everywhere; without the 1/(1 - p)
    factor it does not."""
    q, k, v, _ = _qkv(16, 8, seed=3)
    p, n = 0.3, 400
    mean, std = _mean_over_offsets(oa.attention_forward_dropout, q, k, v, p, n)
    o0, _ = oa.attention_forward(q, k, v, 0.5, False)
    z = np.abs(mean - o0) / (std / math.sqrt(n) + 1e-12)
    assert z.max() < 5.5, z.max()

    def no_rescale(q, k, v, scale, causal, p, seed, offset):  # planted: forgets 1 / (1 - p)
        o, lse = oa.attention_forward_dropout(q, k, v, scale, causal, p, seed, offset)
        return o * (1 - p), lse
    mean_bad, std_bad = _mean_over_offsets(no_rescale, q, k, v, p, n)
    z_bad = np.abs(mean_bad - o0) / (std_bad / math.sqrt(n) + 1e-12)
    assert z_bad.max() > 5.5


def _loss(q, k, v, do, causal, p, seed, offset):
    o, _ = oa.attention_forward_dropout(q, k, v, 0.35, causal, p, seed, offset)
    return float((o * do).sum())


@pytest.mark.parametrize("causal", [False, True])
def test_dropout_backward_matches_finite_differences(causal):
    """For a fixed mask the dropped output is smooth in Q, K, V: central
    differences of L = sum(dO * O) against the analytic gradients."""
    q, k, v, do = _qkv(12, 4, seed=4)
    p, seed, off = 0.3, 5, 9
    grads = oa.attention_backward_dropout(q, k, v, do, 0.35, causal, p, seed, off)
    eps = 1e-6
    for idx, (x, g) in enumerate(zip((q, k, v), grads)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            mi = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[mi] += eps
            xm[mi] -= eps
            args = [q, k, v]
            args[idx] = xp
            lp = _loss(*args, do, causal, p, seed, off)
            args[idx] = xm
            lm = _loss(*args, do, causal, p, seed, off)
            num[mi] = (lp - lm) / (2 * eps)
        assert np.allclose(g, num, rtol=1e-5, atol=1e-7), (idx, np.abs(g - num).max())


def test_planted_mask_in_ds_fails_finite_differences():
    """dS built from the dropped P (instead of P times the dropped dP) is a
    plausible mistake; the finite-difference pin rejects it."""
    q, k, v, do = _qkv(12, 4, seed=6)
    p, seed, off = 0.3, 5, 9
    keep = oa.dropout_keep(0, np.arange(12), np.arange(12), p, seed, off)
    qq, kk, vv, dd = q[0, 0], k[0, 0], v[0, 0], do[0, 0]
    s = oa.attention_scores(qq, kk, 0.35)
    pr, _, _ = oa._three_pass(s, oa._visible(12, 12, False))
    pd = pr * keep * oa.dropout_scale(p)
    dpd = dd @ vv.T
    wrong_ds = pd * (dpd - (pd * dpd).sum(axis=1, keepdims=True))
    wrong_dq = 0.35 * (wrong_ds @ kk)
    right_dq = oa.attention_backward_dropout(q, k, v, do, 0.35, False, p, seed, off)[0][0, 0]
    assert np.abs(wrong_dq - right_dq).max() > 1e-3


def test_planted_head_independent_mask_is_detected():
    """Every head draws its own mask: a mask that ignored the head index
    would make two heads with identical inputs give identical outputs."""
    q, k, v, _ = _qkv(32, 8, seed=7)
    q2, k2, v2 = (np.concatenate([x, x], axis=1) for x in (q, k, v))
    o, _ = oa.attention_forward_dropout(q2, k2, v2, 0.3, False, 0.5, seed=3, offset=0)
    assert np.abs(o[0, 0] - o[0, 1]).max() > 1e-3


def test_packed_dropout_equals_dense_for_equal_lengths():
    """A pack of equal-length sequences drops exactly what the dense batch
    of the same shape drops (sequence s takes batch index s), so its O, LSE
    and gradients equal the dense ones."""
    g = np.random.default_rng(4)
    nseq, H, L, D = 3, 2, 20, 8
    q, k, v, do = (g.standard_normal((nseq, H, L, D)) for _ in range(4))
    packed = [x.transpose(1, 0, 2, 3).reshape(H, nseq * L, D) for x in (q, k, v, do)]
    cu = np.arange(nseq + 1) * L
    for causal in (False, True):
        o_d, l_d = oa.attention_forward_dropout(q, k, v, 0.3, causal, 0.4, seed=9, offset=2)
        o_p, l_p = oa.varlen_forward_dropout(*packed[:3], cu, 0.3, causal, 0.4, seed=9, offset=2)
        assert np.allclose(o_p, o_d.transpose(1, 0, 2, 3).reshape(H, nseq * L, D), atol=1e-13)
        assert np.allclose(l_p, l_d.transpose(1, 0, 2).reshape(H, nseq * L), atol=1e-13)
        g_d = oa.attention_backward_dropout(q, k, v, do, 0.3, causal, 0.4, seed=9, offset=2)
        g_p = oa.varlen_backward_dropout(*packed, cu, 0.3, causal, 0.4, seed=9, offset=2)
        for a, b in zip(g_p, g_d):
            assert np.allclose(a, b.transpose(1, 0, 2, 3).reshape(H, nseq * L, D), atol=1e-12)


def test_packed_dropout_p0_is_plain_and_sequences_get_their_own_masks():
    """p = 0 is plain packed attention; two sequences of one pack with the
    same inputs get different outputs (their masks differ), and a planted
    mistake (every sequence reusing sequence 0's mask) makes them equal."""
    g = np.random.default_rng(5)
    H, L, D = 2, 24, 8
    q1, k1, v1 = (g.standard_normal((H, L, D)) for _ in range(3))
    q, k, v = (np.concatenate([x, x], axis=1) for x in (q1, k1, v1))
    cu = np.array([0, L, 2 * L])
    o0, l0 = oa.varlen_forward_dropout(q, k, v, cu, 0.3, True, 0.0, seed=1, offset=0)
    o_ref, l_ref = oa.varlen_forward(q, k, v, cu, 0.3, True)
    assert np.allclose(o0, o_ref, atol=1e-13) and np.allclose(l0, l_ref, atol=1e-13)
    o, _ = oa.varlen_forward_dropout(q, k, v, cu, 0.3, True, 0.5, seed=1, offset=0)
    assert not np.allclose(o[:, :L], o[:, L:])
    real = oa.dropout_keep

    def same_for_all_sequences(bh, rows, cols, p, seed, offset):
        return real(bh % H, rows, cols, p, seed, offset)

    oa.dropout_keep = same_for_all_sequences
    try:
        o_bad, _ = oa.varlen_forward_dropout(q, k, v, cu, 0.3, True, 0.5, seed=1, offset=0)
    finally:
        oa.dropout_keep = real
    assert np.allclose(o_bad[:, :L], o_bad[:, L:])
