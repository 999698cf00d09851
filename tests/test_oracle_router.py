"""Pins for the oracle's router (oracle/router.py) and permutation (oracle/permute.py):
brute force on tiny inputs, the tie rule, and the routing invariants."""
import itertools
import math

import numpy as np

from oracle import permute as operm
from oracle import router


def test_logits_brute_force():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((3, 5))
    W = rng.standard_normal((5, 4))
    b = rng.standard_normal(4)
    z = router.router_logits(x, W, b)
    for t in range(3):
        for e in range(4):
            ref = sum(x[t, i] * W[i, e] for i in range(5)) + b[e]
            assert abs(z[t, e] - ref) < 1e-12


def test_topk_against_full_sort_and_invariants():
    rng = np.random.default_rng(1)
    for E, k in ((8, 2), (32, 4), (64, 16), (5, 5)):
        z = rng.standard_normal((20, E))
        idx, w, gap = router.route(z, k)
        for t in range(20):
            # brute force: all k-subsets, pick the one with the largest sorted logits
            ranked = sorted(range(E), key=lambda e: (-z[t, e], e))
            assert list(idx[t]) == ranked[:k]
            assert len(set(idx[t])) == k
            s = 1 / (1 + np.exp(-z[t, idx[t]]))
            assert np.allclose(w[t], s / s.sum(), rtol=0, atol=1e-15)
        assert np.all(w > 0)
        assert np.allclose(w.sum(1), 1.0, rtol=0, atol=1e-15)
        if k < E:
            assert np.all(gap >= 0)


def test_tie_rule_lower_index_wins():
    z = np.array([[0.5, 1.0, 1.0, 0.2, 1.0, 0.9]])
    idx, w, gap = router.route(z, 2)
    assert list(idx[0]) == [1, 2]
    assert gap[0] == 0.0
    idx3, _, _ = router.route(z, 3)
    assert list(idx3[0]) == [1, 2, 4]
    # equal logits give equal weights
    assert w[0, 0] == w[0, 1]


def test_selection_by_logit_matches_selection_by_score():
    """sigmoid is monotone: picking by z and by sigmoid(z) agree when scores differ."""
    rng = np.random.default_rng(2)
    z = rng.standard_normal((50, 40)) * 3
    idx, _, _ = router.route(z, 6)
    s = router.sigmoid(z)
    for t in range(50):
        assert set(idx[t]) == set(np.argsort(-s[t], kind="stable")[:6])


def test_k_equals_e_is_a_dense_mixture():
    rng = np.random.default_rng(3)
    z = rng.standard_normal((4, 6))
    idx, w, gap = router.route(z, 6)
    assert np.all(np.isinf(gap))
    s = router.sigmoid(z)
    for t in range(4):
        assert np.allclose(w[t][np.argsort(idx[t])], s[t] / s[t].sum(), atol=1e-15)


def test_permutation_brute_force():
    rng = np.random.default_rng(4)
    T, E, k = 9, 6, 3
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    counts, offsets, perm_tok, inv = operm.permute(idx, E)
    pairs = sorted(((idx[t, j], t, j) for t in range(T) for j in range(k)))
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert np.all(np.diff(offsets) == counts)
    for p, (e, t, j) in enumerate(pairs):
        assert perm_tok[p] == t
        assert inv[t, j] == p
        assert offsets[e] <= p < offsets[e + 1]
    # permute then unpermute is the identity
    vals = rng.standard_normal((T, k))
    permuted = np.empty(T * k)
    permuted[inv.reshape(-1)] = vals.reshape(-1)
    assert np.array_equal(permuted[inv], vals)
    assert sorted(inv.reshape(-1)) == list(range(T * k))


def test_permutation_empty_and_single_expert():
    counts, offsets, perm_tok, inv = operm.permute(np.zeros((0, 2), np.int32), 4)
    assert list(offsets) == [0, 0, 0, 0, 0] and len(perm_tok) == 0
    counts, offsets, perm_tok, inv = operm.permute(np.zeros((5, 1), np.int32), 1)
    assert list(perm_tok) == [0, 1, 2, 3, 4] and list(inv[:, 0]) == [0, 1, 2, 3, 4]


def test_config_closed_forms():
    """The K3 config printed on the pages is consistent with the page totals."""
    import os
    cfg = {}
    for line in open(os.path.join(os.path.dirname(__file__), "golden", "k3_config.txt")):
        if line.strip() and not line.startswith("#"):
            key, val = line.split()
            cfg[key] = val
    E, k = int(cfg["num_experts"]), int(cfg["num_experts_per_token"])
    I, dl = int(cfg["moe_intermediate_size"]), int(cfg["routed_expert_hidden_size"])
    moe_layers = int(cfg["num_hidden_layers"]) - int(cfg["first_k_dense_replace"])
    routed = moe_layers * E * 3 * dl * I
    assert abs(routed / 1e12 - float(cfg["total_params_trillion"])) < 0.1
    assert abs(100.0 * k / E - float(cfg["active_share_percent"])) < 0.05
    assert int(cfg["hidden_size"]) == 2 * dl


# ------------------------------------------------------------------ select-only bias (R20)
def test_select_only_bias_brute_force():
    """Selection by z + b (full sort, lower index on ties), weights from sigmoid(z)."""
    rng = np.random.default_rng(21)
    T, E, k = 7, 12, 4
    z = rng.standard_normal((T, E))
    b = rng.standard_normal(E)
    b[3] = b[5] = 0.25
    z[:, 3] = z[:, 5] = 0.1          # an exact tie on the key, broken by the index
    idx, w, gap = router.route(z, k, select_bias=b)
    for t in range(T):
        key = [(-(z[t, e] + b[e]), e) for e in range(E)]
        sel = [e for _, e in sorted(key)[:k]]
        assert list(idx[t]) == sel
        s = [1.0 / (1.0 + math.exp(-z[t, e])) for e in sel]
        assert np.allclose(w[t], [v / sum(s) for v in s], rtol=1e-15, atol=0)
        keys = sorted((z[t, e] + b[e] for e in range(E)), reverse=True)
        g = 1.0 / (1.0 + math.exp(-keys[k - 1])) - 1.0 / (1.0 + math.exp(-keys[k]))
        assert abs(gap[t] - g) <= 1e-15


def test_select_only_agrees_with_logit_bias_on_selection():
    rng = np.random.default_rng(22)
    z = rng.standard_normal((50, 64))
    b = rng.standard_normal(64)
    i1, w1, _ = router.route(z, 8, select_bias=b)
    i2, w2, _ = router.route(z + b[None, :], 8)
    assert np.array_equal(i1, i2)                 # same key, same experts
    assert not np.allclose(w1, w2)                # weights differ: sigmoid(z) vs sigmoid(z + b)
    i0, w0, g0 = router.route(z, 8, select_bias=np.zeros(64))
    i3, w3, g3 = router.route(z, 8)
    assert np.array_equal(i0, i3) and np.array_equal(w0, w3) and np.array_equal(g0, g3)


def test_select_only_key_in_fp32_when_given_fp32():
    """The key is formed in the logits' own precision, so fp32 logits give fp32 decisions."""
    z = np.array([[1.0, 1.0 + 2.0 ** -23]], dtype=np.float32)
    b = np.array([2.0 ** -24, 0.0], dtype=np.float32)
    # in fp32, 1 + 2^-24 rounds to 1 (ties to even): the keys are (1, 1 + 2^-23), expert 1 wins;
    # in fp64 the keys would be (1 + 2^-24, 1 + 2^-23): expert 1 wins as well, so use a tie
    z2 = np.array([[1.0 + 2.0 ** -23, 1.0]], dtype=np.float32)
    b2 = np.array([0.0, 2.0 ** -23 + 2.0 ** -25], dtype=np.float32)
    idx, _, _ = router.route(z2, 1, select_bias=b2)
    # fp32: 1 + (2^-23 + 2^-25) rounds to 1 + 2^-23, a tie with expert 0, which wins (lower index)
    assert idx[0, 0] == 0
    idx64, _, _ = router.route(z2.astype(np.float64), 1, select_bias=b2.astype(np.float64))
    assert idx64[0, 0] == 1                       # in fp64 the key of expert 1 is larger
    assert router.route(z, 1, select_bias=b)[0][0, 0] == 1


# ------------------------------------------------------------------ Quantile Balancing inputs (R23)
def test_routing_margins_hand_computed():
    # k = 2: the threshold is the 2nd largest logit (2.0)
    z = np.array([[3.0, 1.0, 2.0, 0.0]])
    assert np.array_equal(router.routing_margins(z, 2), [[1.0, -1.0, 0.0, -2.0]])
    # select-only: the key is z + b; with z = 0 the margins are b minus its 2nd largest value
    b = np.array([1.0, 3.0, 2.0, 0.0])
    assert np.array_equal(router.routing_margins(np.zeros((1, 4)), 2, select_bias=b), [[-1.0, 1.0, 0.0, -2.0]])
    # k = E: every expert is selected, the threshold is the smallest key
    assert np.array_equal(router.routing_margins(z, 4), [[3.0, 1.0, 2.0, 0.0]])


def test_routing_margins_agree_with_the_selection():
    """With distinct keys, exactly the selected experts have m >= 0, the k-th selected one
    has m == 0, and m keeps the order of the keys within a token."""
    g = np.random.default_rng(4)
    for T, E, k in ((50, 32, 4), (20, 896, 16), (9, 5, 5)):
        z = g.standard_normal((T, E))
        m = router.routing_margins(z, k)
        idx = router.topk_select(z, k)
        sel = np.zeros((T, E), bool)
        np.put_along_axis(sel, idx.astype(np.int64), True, axis=1)
        assert np.array_equal(m >= 0, sel)
        assert np.all(m[np.arange(T), idx[:, k - 1]] == 0.0)
        assert np.array_equal(np.argsort(-m, axis=1, kind="stable"), np.argsort(-z, axis=1, kind="stable"))


def test_routing_margins_in_fp32_for_fp32_logits():
    """fp32 logits give fp32 margins: each one is the correctly rounded fp32 difference,
    which is what an fp32 kernel computes."""
    g = np.random.default_rng(5)
    z = g.standard_normal((30, 64)).astype(np.float32)
    b = (g.standard_normal(64) * 0.1).astype(np.float32)
    m = router.routing_margins(z, 6, select_bias=b)
    assert m.dtype == np.float32
    key = (z + b).astype(np.float64)                   # fp32 sums, held exactly in fp64
    for t in range(30):
        theta = sorted(key[t], reverse=True)[5]
        for e in range(64):
            assert m[t, e] == np.float32(key[t, e] - theta)   # exact difference, rounded once


def test_quantile_rank_and_quantiles_hand_computed():
    col = np.array([[5.0], [1.0], [3.0], [2.0]])       # sorted: 1, 2, 3, 5
    levels = [0.0, 0.25, 0.26, 0.5, 0.75, 0.99, 1.0]
    assert [router.quantile_rank(q, 4) for q in levels] == [1, 1, 2, 2, 3, 4, 4]
    assert np.array_equal(router.margin_quantiles(col, levels)[:, 0], [1, 1, 2, 2, 3, 5, 5])


def test_margin_quantiles_are_numpys_inverted_cdf_quantiles():
    """The level-q quantile (R23) is numpy's "inverted_cdf" method (the inverse of the
    empirical distribution function), column by column."""
    g = np.random.default_rng(6)
    m = g.standard_normal((257, 40))
    levels = [0.0, 0.01, 1 / 3, 0.5, 0.9, 1 - 16 / 896, 1.0]
    got = router.margin_quantiles(m, levels)
    for i, q in enumerate(levels):
        assert np.array_equal(got[i], np.quantile(m, q, axis=0, method="inverted_cdf"))


def test_margin_quantiles_planted_threshold_mistake_is_caught():
    """Taking the (k+1)-th key as the threshold (a plausible slip) breaks the pin that
    selected experts are exactly those with m >= 0."""
    g = np.random.default_rng(7)
    z = g.standard_normal((40, 32))
    k = 4
    wrong = z - (-np.sort(-z, axis=1))[:, k][:, None]
    idx = router.topk_select(z, k)
    sel = np.zeros(z.shape, bool)
    np.put_along_axis(sel, idx.astype(np.int64), True, axis=1)
    assert not np.array_equal(wrong >= 0, sel)
    assert np.array_equal(router.routing_margins(z, k) >= 0, sel)
