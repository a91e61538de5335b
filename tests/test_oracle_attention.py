"""Pins for the oracle's lightning indexer, top-k selector and core MQA with
sink: closed forms, invariants, brute force and library routines."""
import itertools

import numpy as np
import pytest
from scipy.special import softmax

RNG = np.random.default_rng(11)


# ---------------------------------------------------------------- indexer
def test_index_query_is_linear_map(oracle_lib):
    HI, dI, dc = 3, 8, 16
    W = RNG.standard_normal((HI * dI, dc))
    for c in range(dc):
        e = np.zeros(dc)
        e[c] = 1.0
        # unit latent picks out column c of W
        assert np.array_equal(oracle_lib.index_query(e, W, HI, dI).reshape(-1), W[:, c])


def test_index_scores_unit_query_closed_form(oracle_lib):
    """One head, weight 1, q = e_3: score_s = max(0, k_s[3])."""
    dI = 16
    keys = RNG.standard_normal((50, dI))
    q = np.zeros((1, dI))
    q[0, 3] = 1.0
    sc = oracle_lib.index_scores(q, np.ones(1), keys)
    assert np.array_equal(sc, np.maximum(keys[:, 3], 0.0))
    # negative weight flips the sign, never the ReLU side
    sc2 = oracle_lib.index_scores(q, -2.0 * np.ones(1), keys)
    assert np.array_equal(sc2, -2.0 * np.maximum(keys[:, 3], 0.0))


def test_index_scores_heads_add_and_relu_per_head(oracle_lib):
    dI = 8
    keys = RNG.standard_normal((40, dI))
    q = RNG.standard_normal((2, dI))
    w = np.array([0.7, 1.9])
    both = oracle_lib.index_scores(q, w, keys)
    h0 = oracle_lib.index_scores(q[:1], w[:1], keys)
    h1 = oracle_lib.index_scores(q[1:], w[1:], keys)
    assert np.allclose(both, h0 + h1, atol=1e-14)
    # ReLU is applied per head before the weighted sum: q and -q heads with
    # equal weights give |<q,k>|
    sym = oracle_lib.index_scores(np.stack([q[0], -q[0]]), np.ones(2), keys)
    assert np.allclose(sym, np.abs(keys @ q[0]), atol=1e-14)
    # nonnegative weights -> nonnegative scores
    assert np.all(oracle_lib.index_scores(q, np.abs(w), keys) >= 0)


# ---------------------------------------------------------------- top-k
def test_topk_brute_force(oracle_lib):
    for n, k in [(10, 3), (64, 64), (100, 7), (5, 8), (0, 4), (1, 1)]:
        sc = np.round(RNG.standard_normal(n), 1)            # plenty of ties
        got = oracle_lib.topk(sc, k)
        ranked = sorted(range(n), key=lambda i: (-sc[i], i))[:k]
        want = sorted(ranked) + [-1] * (k - min(n, k))
        assert list(got) == want, (n, k)


def test_topk_all_equal_takes_lowest_indices(oracle_lib):
    got = oracle_lib.topk(np.zeros(20), 5)
    assert list(got) == [0, 1, 2, 3, 4]


def test_topk_is_a_set_of_maximal_scores(oracle_lib):
    sc = RNG.standard_normal(1000)
    got = oracle_lib.topk(sc, 100)
    assert np.all(np.diff(got) > 0)
    chosen = set(got.tolist())
    worst_in = min(sc[i] for i in chosen)
    best_out = max(sc[i] for i in range(1000) if i not in chosen)
    assert worst_in >= best_out


# ---------------------------------------------------------------- attention
def _setup(H=4, D=128, n=20, t=300):
    q = RNG.standard_normal((H, D))
    g = 1 + 0.1 * RNG.standard_normal(D)
    rows = RNG.standard_normal((n, D))
    sink = RNG.standard_normal(H)
    return q, g, rows, sink, t


def test_attend_matches_softmax_with_sink_as_extra_logit(oracle_lib):
    """The sink is one more logit whose value vector is zero: the output is
    softmax([z, s_1..s_n])[1:] @ rows (scipy's softmax as the library routine)."""
    q, g, rows, sink, t = _setup()
    out, share = oracle_lib.attend(q, g, t, rows, sink)
    for h in range(q.shape[0]):
        qh = oracle_lib.rope(oracle_lib.rmsnorm(q[h], g), t)
        logits = np.concatenate([[sink[h]], rows @ qh / np.sqrt(q.shape[1])])
        p = softmax(logits)
        assert np.allclose(out[h], p[1:] @ rows, atol=1e-13)
        assert abs(share[h] - p[0]) < 1e-15


def test_attend_sink_to_minus_inf_is_plain_softmax(oracle_lib):
    q, g, rows, _, t = _setup()
    out, share = oracle_lib.attend(q, g, t, rows, np.full(q.shape[0], -1e30))
    assert np.all(share == 0.0)
    for h in range(q.shape[0]):
        qh = oracle_lib.rope(oracle_lib.rmsnorm(q[h], g), t)
        p = softmax(rows @ qh / np.sqrt(q.shape[1]))
        assert np.allclose(out[h], p @ rows, atol=1e-13)


def test_attend_weights_and_sink_share_sum_to_one(oracle_lib):
    """With every row = e_d (unit vectors), out[h, d] is the weight p_d, so
    sum_d out[h,d] + sink_share[h] == 1."""
    D = 128
    rows = np.eye(D)[:37]
    q = RNG.standard_normal((3, D))
    out, share = oracle_lib.attend(q, np.ones(D), 999, rows, RNG.standard_normal(3))
    assert np.allclose(out.sum(axis=1) + share, 1.0, atol=1e-12)
    assert np.all(out[:, 37:] == 0)


def test_attend_single_row_returns_row(oracle_lib):
    q, g, rows, _, t = _setup(n=1)
    out, share = oracle_lib.attend(q, g, t, rows, np.full(q.shape[0], -1e30))
    assert np.allclose(out, np.broadcast_to(rows[0], out.shape), atol=1e-14)


def test_attend_large_sink_drains_attention(oracle_lib):
    q, g, rows, _, t = _setup()
    out_lo, sh_lo = oracle_lib.attend(q, g, t, rows, np.zeros(q.shape[0]))
    out_hi, sh_hi = oracle_lib.attend(q, g, t, rows, np.full(q.shape[0], 40.0))
    assert np.all(sh_hi > sh_lo) and np.all(sh_hi > 1 - 1e-12)
    assert np.abs(out_hi).max() < 1e-12


def test_attend_order_of_rows_does_not_matter(oracle_lib):
    q, g, rows, sink, t = _setup()
    perm = RNG.permutation(rows.shape[0])
    a, _ = oracle_lib.attend(q, g, t, rows, sink)
    b, _ = oracle_lib.attend(q, g, t, rows[perm], sink)
    assert np.allclose(a, b, atol=1e-13)


def test_attend_uses_query_position(oracle_lib):
    """Rotating the query by t and every row by the same shift keeps the
    logits (RoPE relative-position property), so the output of rows rotated
    by +delta at query t+delta equals the rotated output."""
    q, g, rows, sink, t = _setup(D=128)
    # rows whose nope part is zero: then rotation acts on all of them
    rows[:, :64] = 0.0
    a, _ = oracle_lib.attend(q, g, t, rows, sink)
    shifted = np.stack([oracle_lib.rope(r, 50) for r in rows])
    b, _ = oracle_lib.attend(q, g, t + 50, shifted, sink)
    assert np.allclose(np.stack([oracle_lib.rope(x, 50) for x in a]), b, atol=1e-12)
