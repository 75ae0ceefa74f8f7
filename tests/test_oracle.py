"""Pins for the fp64 oracle: closed forms, invariants, brute force and
library cross-checks that do not reuse the oracle's own code.

Each pin is written as a function of the oracle's forward/backward so that
``test_pins_catch_planted_mistakes`` can run the same pins against copies of
the oracle with a deliberate mistake planted in them (on the CPU) and show
that every such mistake fails at least one pin.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as oa
from exact_tiled_attention_31_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed=0):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------
# brute force: pure-Python loops over the textbook definition (tiny inputs)
# --------------------------------------------------------------------------

def brute_forward(q, k, v, scale, causal):
    nq, d = len(q), len(q[0])
    o, lse = [], []
    for i in range(nq):
        keys = [j for j in range(len(k)) if (not causal or j <= i)]
        s = [scale * sum(q[i][t] * k[j][t] for t in range(d)) for j in keys]
        mx = max(s)
        w = [math.exp(x - mx) for x in s]
        tot = math.fsum(w)
        o.append([math.fsum(w[n] * v[j][c] for n, j in enumerate(keys)) / tot
                  for c in range(len(v[0]))])
        lse.append(mx + math.log(tot))
    return np.array(o), np.array(lse)


# --------------------------------------------------------------------------
# pins (each returns normally or raises AssertionError)
# --------------------------------------------------------------------------

def pin_q_zero(fwd, bwd):
    """Q = 0: every score is 0, so O is the mean of the visible V rows
    (prefix means under the causal mask) and LSE = ln(#visible)."""
    r = _rng(1)
    S, D = 37, 8
    q = np.zeros((S, D))
    k, v = r.standard_normal((S, D)), r.standard_normal((S, D))
    o, lse = fwd(q, k, v, 0.3, False)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(0), o.shape), atol=1e-13)
    np.testing.assert_allclose(lse, np.full(S, math.log(S)), atol=1e-13)
    o, lse = fwd(q, k, v, 0.3, True)
    pref = np.cumsum(v, 0) / np.arange(1, S + 1)[:, None]
    np.testing.assert_allclose(o, pref, atol=1e-13)
    np.testing.assert_allclose(lse, np.log(np.arange(1, S + 1)), atol=1e-13)


def pin_dominant_score(fwd, bwd):
    """One key aligned with the query and far above the rest selects its V row;
    LSE then equals that single score (up to exp(-gap))."""
    r = _rng(2)
    S, D = 16, 8
    k = 0.01 * r.standard_normal((S, D))
    v = r.standard_normal((S, D))
    q = np.zeros((S, D))
    target = 5
    q[:, 0] = 1.0
    k[target, 0] = 400.0
    o, lse = fwd(q, k, v, 0.25, False)
    np.testing.assert_allclose(o, np.broadcast_to(v[target], o.shape), atol=1e-12)
    s_star = 0.25 * (q @ k[target])
    np.testing.assert_allclose(lse, s_star, atol=1e-12)
    # causal: rows before the target cannot see it, rows from it on do
    o, _ = fwd(q, k, v, 0.25, True)
    np.testing.assert_allclose(o[target:], np.broadcast_to(v[target], (S - target, D)), atol=1e-12)
    assert np.abs(o[:target] - v[target]).max() > 0.1


def pin_probs_sum_to_one(fwd, bwd, probs=None):
    probs = probs or oa.attention_probs
    r = _rng(3)
    q, k = r.standard_normal((29, 16)), r.standard_normal((29, 16))
    for causal in (False, True):
        p = probs(q, k, 0.25, causal)
        np.testing.assert_allclose(p.sum(1), 1.0, atol=1e-14)
        assert (p >= 0).all()
        if causal:
            assert np.all(np.triu(p, 1) == 0)


def pin_permutation(fwd, bwd):
    """Non-causal: permuting K and V rows together leaves O and LSE unchanged;
    permuting Q rows permutes O and LSE the same way."""
    r = _rng(4)
    S, D = 23, 16
    q, k, v = (r.standard_normal((S, D)) for _ in range(3))
    o, lse = fwd(q, k, v, 0.25, False)
    perm = r.permutation(S)
    o2, lse2 = fwd(q, k[perm], v[perm], 0.25, False)
    np.testing.assert_allclose(o2, o, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, atol=1e-13)
    o3, lse3 = fwd(q[perm], k, v, 0.25, False)
    np.testing.assert_allclose(o3, o[perm], atol=1e-13)
    np.testing.assert_allclose(lse3, lse[perm], atol=1e-13)


def pin_key_shift(fwd, bwd):
    """Adding c to every key adds scale*q_i.c to every score of row i: O is
    unchanged and LSE moves by exactly that amount (causal too)."""
    r = _rng(5)
    S, D = 19, 8
    q, k, v = (r.standard_normal((S, D)) for _ in range(3))
    c = r.standard_normal(D)
    for causal in (False, True):
        o, lse = fwd(q, k, v, 0.5, causal)
        o2, lse2 = fwd(q, k + c, v, 0.5, causal)
        np.testing.assert_allclose(o2, o, atol=1e-12)
        np.testing.assert_allclose(lse2, lse + 0.5 * (q @ c), atol=1e-12)


def pin_affine_v(fwd, bwd):
    """Rows of P sum to one, so O(a V + b) = a O + b."""
    r = _rng(6)
    S, D = 21, 8
    q, k, v = (r.standard_normal((S, D)) for _ in range(3))
    b = r.standard_normal(D)
    for causal in (False, True):
        o, _ = fwd(q, k, v, 0.25, causal)
        o2, _ = fwd(q, k, 3.0 * v + b, 0.25, causal)
        np.testing.assert_allclose(o2, 3.0 * o + b, atol=1e-12)


def pin_brute_force(fwd, bwd):
    """Pure-Python loops over the definition on tiny inputs."""
    r = _rng(7)
    for S, D, causal in ((5, 3, False), (6, 4, True), (1, 2, True)):
        q, k, v = (r.standard_normal((S, D)) for _ in range(3))
        o, lse = fwd(q, k, v, 0.7, causal)
        ob, lseb = brute_forward(q.tolist(), k.tolist(), v.tolist(), 0.7, causal)
        np.testing.assert_allclose(o, ob, atol=1e-13)
        np.testing.assert_allclose(lse, lseb, atol=1e-13)


def pin_torch_fp64(fwd, bwd):
    """Library cross-check: torch's SDPA and autograd in fp64 on the CPU."""
    r = _rng(8)
    S, D = 33, 16
    for causal in (False, True):
        q, k, v, do = (r.standard_normal((S, D)) for _ in range(4))
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        to = torch.nn.functional.scaled_dot_product_attention(
            tq[None], tk[None], tv[None], is_causal=causal, scale=0.25)[0]
        to.backward(torch.tensor(do))
        o, _ = fwd(q, k, v, 0.25, causal)
        np.testing.assert_allclose(o, to.detach().numpy(), atol=1e-12)
        dq, dk, dv = bwd(q, k, v, do, 0.25, causal)
        np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-12)
        np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-12)
        np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-12)


def pin_finite_differences(fwd, bwd):
    """Central differences of L = sum(dO * O) on tiny shapes."""
    r = _rng(9)
    S, D, h = 6, 3, 1e-6
    for causal in (False, True):
        q, k, v, do = (r.standard_normal((S, D)) for _ in range(4))
        grads = bwd(q, k, v, do, 0.6, causal)
        for which, g in zip(range(3), grads):
            args = [q, k, v]
            num = np.zeros_like(args[which])
            for idx in np.ndindex(*num.shape):
                plus = [a.copy() for a in args]
                minus = [a.copy() for a in args]
                plus[which][idx] += h
                minus[which][idx] -= h
                lp = (fwd(*plus, 0.6, causal)[0] * do).sum()
                lm = (fwd(*minus, 0.6, causal)[0] * do).sum()
                num[idx] = (lp - lm) / (2 * h)
            np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-7)


def pin_grad_invariants(fwd, bwd):
    """sum_j dK_j = 0 (each row of dS sums to zero), and with Q = 0 every
    visible P_ij is 1/n_i, so dV_j = sum_{i sees j} dO_i / n_i."""
    r = _rng(10)
    S, D = 17, 8
    for causal in (False, True):
        q, k, v, do = (r.standard_normal((S, D)) for _ in range(4))
        _, dk, _ = bwd(q, k, v, do, 0.4, causal)
        np.testing.assert_allclose(dk.sum(0), 0.0, atol=1e-12)
        _, _, dv = bwd(np.zeros((S, D)), k, v, do, 0.4, causal)
        if causal:
            expect = np.array([sum(do[i] / (i + 1) for i in range(j, S)) for j in range(S)])
        else:
            expect = np.broadcast_to(do.sum(0) / S, (S, D))
        np.testing.assert_allclose(dv, expect, atol=1e-12)


PINS = [pin_q_zero, pin_dominant_score, pin_probs_sum_to_one, pin_permutation,
        pin_key_shift, pin_affine_v, pin_brute_force, pin_torch_fp64,
        pin_finite_differences, pin_grad_invariants]


def _oracle_fwd(q, k, v, scale, causal):
    return oa.attention_forward(q, k, v, scale, causal)


def _oracle_bwd(q, k, v, do, scale, causal):
    return oa.attention_backward(q, k, v, do, scale, causal)


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_oracle_pins(pin):
    pin(_oracle_fwd, _oracle_bwd)


# --------------------------------------------------------------------------
# the one-pass (online) restatement equals the three-pass definition
# --------------------------------------------------------------------------

def test_online_equals_three_pass_page_check():
    """The pages' own check (seed 42, B=2 H=8 N=512 D=64, block 128) bounds
    the online-vs-standard difference; in fp64 both agree to ~1e-13."""
    with open(os.path.join(GOLDEN, "page_checks.json")) as f:
        chk = json.load(f)["online_vs_standard"]
    B, H, N, D = chk["shape"]
    t = inputs.make_dense(B, H, N, D, dtype="bf16", seed=chk["seed"])
    worst = 0.0
    for b in range(B):
        for h in (0, H - 1):
            for causal in (False, True):
                o1, l1 = oa.attention_forward(t["q"][b, h], t["k"][b, h], t["v"][b, h],
                                              1 / math.sqrt(D), causal)
                o2, l2 = oa.attention_forward_online(t["q"][b, h], t["k"][b, h], t["v"][b, h],
                                                     1 / math.sqrt(D), causal, block=chk["block"])
                worst = max(worst, np.abs(o1 - o2).max(), np.abs(l1 - l2).max())
    assert worst < chk["max_diff_bound"]
    assert worst < 1e-12


def test_online_ragged_blocks():
    r = _rng(11)
    q, k, v = (r.standard_normal((45, 8)) for _ in range(3))
    for causal in (False, True):
        for block in (1, 7, 16, 64):
            o1, l1 = oa.attention_forward(q, k, v, 0.3, causal)
            o2, l2 = oa.attention_forward_online(q, k, v, 0.3, causal, block=block)
            np.testing.assert_allclose(o2, o1, atol=1e-13)
            np.testing.assert_allclose(l2, l1, atol=1e-13)


# --------------------------------------------------------------------------
# batched / varlen / row-subset entry points agree with the per-head form
# --------------------------------------------------------------------------

def test_batched_matches_per_head_and_rows():
    t = inputs.make_dense(2, 3, 40, 16, dtype="fp16", seed=3, with_do=True)
    o, lse = oa.attention_forward(t["q"], t["k"], t["v"], 0.25, True)
    dq, dk, dv = oa.attention_backward(t["q"], t["k"], t["v"], t["do"], 0.25, True)
    for b in range(2):
        for h in range(3):
            oh, lh = oa.attention_forward(t["q"][b, h], t["k"][b, h], t["v"][b, h], 0.25, True)
            np.testing.assert_array_equal(o[b, h], oh)
            np.testing.assert_array_equal(lse[b, h], lh)
            g = oa.attention_backward(t["q"][b, h], t["k"][b, h], t["v"][b, h], t["do"][b, h], 0.25, True)
            np.testing.assert_array_equal(dq[b, h], g[0])
            np.testing.assert_array_equal(dk[b, h], g[1])
            np.testing.assert_array_equal(dv[b, h], g[2])
    rows = [0, 5, 39]
    orow, lrow = oa.attention_forward_rows(t["q"], t["k"], t["v"], 0.25, True, 1, 2, rows)
    np.testing.assert_allclose(orow, o[1, 2, rows], atol=1e-14)
    np.testing.assert_allclose(lrow, lse[1, 2, rows], atol=1e-14)


def test_varlen_is_block_diagonal():
    """A packed batch equals each sequence run on its own, and differs from
    running the whole pack as one sequence (sequences must not see each other)."""
    t = inputs.make_varlen(4, 3, 9, 2, 8, dtype="bf16", seed=5, with_do=True)
    cu = t["cu_seqlens"].tolist()
    o, lse = oa.varlen_forward(t["q"], t["k"], t["v"], t["cu_seqlens"], 0.3, True)
    g = oa.varlen_backward(t["q"], t["k"], t["v"], t["do"], t["cu_seqlens"], 0.3, True)
    for h in range(2):
        for a, b in zip(cu[:-1], cu[1:]):
            ob, lb = brute_forward(oa.to_f64(t["q"][h, a:b]).tolist(), oa.to_f64(t["k"][h, a:b]).tolist(),
                                   oa.to_f64(t["v"][h, a:b]).tolist(), 0.3, True)
            np.testing.assert_allclose(o[h, a:b], ob, atol=1e-13)
            np.testing.assert_allclose(lse[h, a:b], lb, atol=1e-13)
            gd = oa.attention_backward(t["q"][h, a:b], t["k"][h, a:b], t["v"][h, a:b], t["do"][h, a:b], 0.3, True)
            for x, y in zip(g, gd):
                np.testing.assert_allclose(x[h, a:b], y, atol=1e-13)
    whole, _ = oa.attention_forward(t["q"][0], t["k"][0], t["v"][0], 0.3, True)
    assert np.abs(whole - o[0]).max() > 1e-3


def test_inputs_are_seeded_and_rounded():
    a = inputs.make_dense(1, 2, 8, 4, dtype="bf16", seed=42, qk_mult=8.0)
    b = inputs.make_dense(1, 2, 8, 4, dtype="bf16", seed=42, qk_mult=8.0)
    for key in ("q", "k", "v"):
        assert torch.equal(a[key], b[key])
        assert a[key].dtype == torch.bfloat16
    c = inputs.make_dense(1, 2, 8, 4, dtype="bf16", seed=42)
    assert torch.equal(a["q"].float(), 8.0 * c["q"].float())   # power-of-two scaling is exact
    assert torch.equal(a["v"], c["v"])
    vl = inputs.make_varlen(32, 128, 4096, 1, 8, seed=42)
    assert all(128 <= L <= 4096 for L in vl["lengths"])
    assert vl["cu_seqlens"][-1] == vl["total"] == sum(vl["lengths"])


def test_flop_convention():
    f, b = oa.flop_count([4096], 32, 128, True)
    assert f == pytest.approx(4 * 32 * 4096 ** 2 * 128 / 2)
    assert b == pytest.approx(2.5 * f)


# --------------------------------------------------------------------------
# planted mistakes: every one must fail at least one pin
# --------------------------------------------------------------------------

def _mut_mask_off_by_one(nq, nk, causal, q_rows=None):
    rows = np.arange(nq) if q_rows is None else np.asarray(q_rows)
    cols = np.arange(nk)
    if causal:
        return cols[None, :] < rows[:, None] + (rows[:, None] == 0)
    return np.ones((rows.shape[0], nk), dtype=bool)


def _mut_no_scale(q, k, scale):
    return q @ k.T


def _mut_transposed_scores(q, k, scale):
    return scale * (q @ k.T).T


def _mut_lse_log2(s, vis):
    p, m, l = _orig_three_pass(s, vis)
    return p, m, l / math.e * 2.0


def _mut_no_normalise(s, vis):
    p, m, l = _orig_three_pass(s, vis)
    return p * l[:, None] / (l[:, None] + 1.0), m, l


def _mut_bwd_sign(q, k, v, do, scale, causal):
    dq, dk, dv, o = _orig_head_backward(q, k, v, do, scale, causal)
    s = oa.attention_scores(q, k, scale)
    p, _, _ = _orig_three_pass(s, oa._visible(q.shape[0], k.shape[0], causal))
    dp = do @ v.T
    ds = p * (dp + (p * dp).sum(1)[:, None])
    return scale * ds @ k, scale * ds.T @ q, dv, o


def _mut_dk_no_scale(q, k, v, do, scale, causal):
    dq, dk, dv, o = _orig_head_backward(q, k, v, do, scale, causal)
    return dq, dk / scale, dv, o


def _mut_dv_transposed(q, k, v, do, scale, causal):
    dq, dk, dv, o = _orig_head_backward(q, k, v, do, scale, causal)
    s = oa.attention_scores(q, k, scale)
    p, _, _ = _orig_three_pass(s, oa._visible(q.shape[0], k.shape[0], causal))
    return dq, dk, p @ do, o


_orig_three_pass = oa._three_pass
_orig_head_backward = oa._head_backward

MUTANTS = {
    "causal_off_by_one": ("_visible", _mut_mask_off_by_one),
    "missing_scale": ("attention_scores", _mut_no_scale),
    "transposed_scores": ("attention_scores", _mut_transposed_scores),
    "wrong_lse": ("_three_pass", _mut_lse_log2),
    "unnormalised": ("_three_pass", _mut_no_normalise),
    "bwd_sign": ("_head_backward", _mut_bwd_sign),
    "dk_missing_scale": ("_head_backward", _mut_dk_no_scale),
    "dv_transposed": ("_head_backward", _mut_dv_transposed),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(oa, attr, fn)
    failed = []
    for pin in PINS:
        try:
            pin(_oracle_fwd, _oracle_bwd)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"planted mistake {name} passed every pin"


# ---------------------------------------------------------------- decode
def _decode_inputs(B=2, Hq=8, Hkv=2, L=37, D=8, seed=3):
    g = np.random.default_rng(seed)
    q = g.standard_normal((B, Hq, D))
    k = g.standard_normal((B, Hkv, L, D))
    v = g.standard_normal((B, Hkv, L, D))
    lens = np.array([L, 5][:B] + [L] * max(0, B - 2))
    return q, k, v, lens


def test_decode_is_the_last_row_of_causal_attention():
    """A decode step is the last query row of causal attention over the
    sequence's keys (new token at the end sees every cached key)."""
    q, k, v, lens = _decode_inputs(B=2, Hq=4, Hkv=4)
    o, lse = oa.decode_forward(q, k, v, lens, 0.3)
    for b in range(2):
        L = lens[b]
        for h in range(4):
            qq = np.concatenate([np.zeros((L - 1, q.shape[-1])), q[b, h][None]], axis=0)
            # brute force: explicit exp/sum over the visible keys of the last row
            s = [0.3 * float(q[b, h] @ k[b, h, j]) for j in range(L)]
            mx = max(s)
            w = [math.exp(x - mx) for x in s]
            ref = sum(wi * v[b, h, j] for j, wi in enumerate(w)) / sum(w)
            assert np.allclose(o[b, h], ref, atol=1e-12)
            assert abs(lse[b, h] - (mx + math.log(sum(w)))) < 1e-12
            ob, lb = oa.attention_forward(qq, k[b, h, :L], v[b, h, :L], 0.3, True)
            assert np.allclose(ob[-1], o[b, h], atol=1e-12) and abs(lb[-1] - lse[b, h]) < 1e-12


def test_decode_gqa_equals_repeated_kv_heads():
    q, k, v, lens = _decode_inputs(B=2, Hq=8, Hkv=2)
    o, lse = oa.decode_forward(q, k, v, lens, 0.25)
    o2, lse2 = oa.decode_forward(q, np.repeat(k, 4, axis=1), np.repeat(v, 4, axis=1), lens, 0.25)
    assert np.allclose(o, o2, atol=1e-13) and np.allclose(lse, lse2, atol=1e-13)


def test_decode_q_zero_is_mean_of_visible_values():
    q, k, v, lens = _decode_inputs(B=2, Hq=4, Hkv=1)
    o, lse = oa.decode_forward(np.zeros_like(q), k, v, lens, 0.5)
    for b in range(2):
        assert np.allclose(o[b], v[b, 0, :lens[b]].mean(axis=0), atol=1e-13)
        assert np.allclose(lse[b], math.log(lens[b]), atol=1e-13)


def test_merge_of_split_keys_equals_the_whole():
    """Splitting the cached keys into disjoint ranges and merging the
    per-range (O, LSE) gives the unsplit result; an empty range weighs 0."""
    q, k, v, lens = _decode_inputs(B=1, Hq=2, Hkv=2, L=50)
    o, lse = oa.decode_forward(q, k, v, lens, 0.4)
    cuts = [0, 7, 7, 31, 50]  # includes an empty range
    parts_o, parts_l = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        if b > a:
            po, pl = oa.decode_forward(q, k[:, :, a:b], v[:, :, a:b], [b - a], 0.4)
        else:
            po, pl = np.zeros_like(o), np.full(lse.shape, -np.inf)
        parts_o.append(po)
        parts_l.append(pl)
    mo, ml = oa.merge_partials(np.stack(parts_o), np.stack(parts_l))
    assert np.allclose(mo, o, atol=1e-13) and np.allclose(ml, lse, atol=1e-13)


def test_decode_planted_mistakes_fail():
    """A decode that reads the wrong KV head, or the keys past seq_lens, is caught."""
    q, k, v, lens = _decode_inputs(B=2, Hq=8, Hkv=2)
    o, _ = oa.decode_forward(q, k, v, lens, 0.25)
    wrong_head = np.concatenate([k[:, 1:], k[:, :1]], axis=1)
    o_bad, _ = oa.decode_forward(q, wrong_head, v, lens, 0.25)
    assert not np.allclose(o, o_bad, atol=1e-6)
    o_all, _ = oa.decode_forward(q, k, v, [k.shape[2]] * 2, 0.25)
    assert not np.allclose(o[1], o_all[1], atol=1e-6)  # sequence 1 has only 5 valid keys
