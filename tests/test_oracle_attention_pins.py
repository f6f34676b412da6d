"""Pins of the fp64 attention oracle (oracle/attention.py) to things other than
itself: the hand-worked two-token closed forms, torch's scaled-dot-product
attention routine in fp64, a scalar brute force, the invariants the TSP
schedule must keep (any P, any key/value visiting order, any parameter-shard
order), and special cases with known answers (causal first row, uniform and
one-hot attention)."""
import json
import math
import os
import random

import numpy as np
import pytest
import torch

from oracle import attention as A

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "attention_2tok_closed_form.json")


def sig(z):
    return 1.0 / (1.0 + math.exp(-z))


def ev(grid):
    ns = {"sig": sig, "__builtins__": {}}
    return np.array([[eval(e, ns) for e in row] for row in grid], dtype=np.float64)


@pytest.fixture(scope="module")
def g2():
    with open(GOLDEN) as fh:
        return json.load(fh)


def _inp(g2):
    i = g2["inputs"]
    return [np.array(i[k], float) for k in ("X", "Wq", "Wk", "Wv", "Wo")]


def rel(a, b):
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


def rand_block(n, d, heads, seed, w_std=0.4):
    r = np.random.default_rng(seed)
    X = r.standard_normal((n, d))
    W = [r.standard_normal((d, d)) * w_std for _ in range(4)]
    return X, *W


# ---------------------------------------------------------------------------
# the hand-worked closed forms


def test_golden_numbers_match_their_expressions(g2):
    for form in ("plain", "causal"):
        for key, ent in g2[form].items():
            np.testing.assert_allclose(ev(ent["expr"]), np.array(ent["value"]), rtol=0, atol=1e-15,
                                       err_msg=f"{form}.{key}")


@pytest.mark.parametrize("causal", [False, True])
def test_two_token_block(g2, causal):
    X, Wq, Wk, Wv, Wo = _inp(g2)
    form = g2["causal" if causal else "plain"]
    Y = A.attention_forward(X, Wq, Wk, Wv, Wo, 2, causal)
    np.testing.assert_allclose(Y, ev(form["Y"]["expr"]), rtol=1e-15, atol=1e-15)
    O = A.attention_core(X @ Wq, X @ Wk, X @ Wv, 2, causal)
    np.testing.assert_allclose(O, ev(form["O"]["expr"]), rtol=1e-15, atol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
def test_two_token_tsp_schedule(g2, causal):
    """P = 2: one token per sequence shard and one head per parameter shard;
    either parameter-shard order and either ring direction."""
    X, Wq, Wk, Wv, Wo = _inp(g2)
    form = g2["causal" if causal else "plain"]
    for order in (A.ring_order, A.reverse_ring_order):
        for go in ([0, 1], [1, 0]):
            Y = A.attention_tsp(X, Wq, Wk, Wv, Wo, 2, 2, causal, order=order, group_order=go)
            np.testing.assert_allclose(Y, ev(form["Y"]["expr"]), rtol=1e-15, atol=1e-15)
    O = A.attention_core_tsp(X @ Wq, X @ Wk, X @ Wv, 2, 2, causal)
    np.testing.assert_allclose(O, ev(form["O"]["expr"]), rtol=1e-15, atol=1e-15)


def test_two_token_partials_sum_to_the_output(g2):
    """Each parameter shard's partial output is its head's O times its rows of
    W_o ("Tensor Parallelism: Splitting the Math": output projection split by
    rows, one sum at the end)."""
    X, Wq, Wk, Wv, Wo = _inp(g2)
    p = g2["plain"]
    O = A.attention_core(X @ Wq, X @ Wk, X @ Wv, 2)
    for w in (0, 1):
        c = slice(2 * w, 2 * w + 2)
        np.testing.assert_allclose(O[:, c] @ Wo[c, :], ev(p[f"partial_{w}"]["expr"]), rtol=1e-15,
                                   atol=1e-15)
    np.testing.assert_allclose(ev(p["partial_0"]["expr"]) + ev(p["partial_1"]["expr"]),
                               ev(p["Y"]["expr"]), rtol=1e-15, atol=1e-15)


# ---------------------------------------------------------------------------
# a library routine and a scalar brute force


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,d,heads", [(7, 8, 2), (33, 16, 4), (64, 24, 3)])
def test_core_equals_torch_sdpa_fp64(n, d, heads, causal):
    X, Wq, Wk, Wv, _ = rand_block(n, d, heads, seed=n + d + heads)
    Q, K, V = X @ Wq, X @ Wk, X @ Wv
    dh = d // heads
    t = lambda M: torch.from_numpy(M).view(n, heads, dh).transpose(0, 1)  # [heads][n][dh]
    ref = torch.nn.functional.scaled_dot_product_attention(t(Q), t(K), t(V), is_causal=causal)
    ref = ref.transpose(0, 1).reshape(n, d).numpy()
    O = A.attention_core(Q, K, V, heads, causal)
    assert rel(O, ref) <= 1e-13
    Ot = A.attention_core_tsp(Q, K, V, heads, 1, causal)
    assert rel(Ot, ref) <= 1e-13


def _brute(X, Wq, Wk, Wv, Wo, heads, causal):
    n, d = len(X), len(X[0])
    dh = d // heads
    proj = lambda W: [[sum(X[i][k] * W[k][j] for k in range(d)) for j in range(d)] for i in range(n)]
    Q, K, V = proj(Wq), proj(Wk), proj(Wv)
    O = [[0.0] * d for _ in range(n)]
    for h in range(heads):
        for i in range(n):
            keys = [j for j in range(n) if not (causal and j > i)]
            s = {j: sum(Q[i][h * dh + e] * K[j][h * dh + e] for e in range(dh)) / math.sqrt(dh)
                 for j in keys}
            mx = max(s.values())
            w = {j: math.exp(s[j] - mx) for j in keys}
            tot = sum(w.values())
            for e in range(dh):
                O[i][h * dh + e] = sum(w[j] * V[j][h * dh + e] for j in keys) / tot
    return np.array([[sum(O[i][k] * Wo[k][j] for k in range(d)) for j in range(d)]
                     for i in range(n)])


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,d,heads,P", [(4, 4, 2, 2), (6, 6, 3, 3), (8, 4, 2, 2)])
def test_brute_force_tiny(n, d, heads, P, causal):
    X, Wq, Wk, Wv, Wo = rand_block(n, d, heads, seed=100 + n * d, w_std=0.8)
    ref = _brute(X.tolist(), Wq.tolist(), Wk.tolist(), Wv.tolist(), Wo.tolist(), heads, causal)
    assert rel(A.attention_forward(X, Wq, Wk, Wv, Wo, heads, causal), ref) <= 1e-13
    assert rel(A.attention_tsp(X, Wq, Wk, Wv, Wo, heads, P, causal), ref) <= 1e-13


# ---------------------------------------------------------------------------
# invariants of the TSP schedule


@pytest.mark.parametrize("causal", [False, True])
def test_tsp_independent_of_P_and_equal_to_plain(causal):
    n, d, heads = 48, 32, 8
    X, Wq, Wk, Wv, Wo = rand_block(n, d, heads, seed=7)
    ref = A.attention_forward(X, Wq, Wk, Wv, Wo, heads, causal)
    Y1 = A.attention_tsp(X, Wq, Wk, Wv, Wo, heads, 1, causal)
    assert rel(Y1, ref) <= 1e-13
    for P in (2, 4, 8):
        assert rel(A.attention_tsp(X, Wq, Wk, Wv, Wo, heads, P, causal), ref) <= 1e-12


def _perm_order(P, seed):
    r = random.Random(seed)
    perms = {}
    for s in range(P):
        rest = [u for u in range(P) if u != s]
        r.shuffle(rest)
        perms[s] = [s] + rest

    def order(s, t, P_):
        return perms[s][t]
    return order


@pytest.mark.parametrize("causal", [False, True])
def test_tsp_independent_of_visiting_and_shard_order(causal):
    n, d, heads, P = 40, 16, 4, 4
    X, Wq, Wk, Wv, Wo = rand_block(n, d, heads, seed=9)
    ref = A.attention_forward(X, Wq, Wk, Wv, Wo, heads, causal)
    for order in (A.ring_order, A.reverse_ring_order, _perm_order(P, 3)):
        for go in (None, [3, 1, 0, 2]):
            Y = A.attention_tsp(X, Wq, Wk, Wv, Wo, heads, P, causal, order=order, group_order=go)
            assert rel(Y, ref) <= 1e-12
    Q, K, V = X @ Wq, X @ Wk, X @ Wv
    Oref = A.attention_core(Q, K, V, heads, causal)
    for order in (A.ring_order, A.reverse_ring_order, _perm_order(P, 4)):
        assert rel(A.attention_core_tsp(Q, K, V, heads, P, causal, order), Oref) <= 1e-12


def test_ring_visits_every_shard_once_starting_at_its_own():
    for P in (1, 2, 3, 8):
        for s in range(P):
            seen = [A.ring_order(s, t, P) for t in range(P)]
            assert seen[0] == s and sorted(seen) == list(range(P))
            assert seen[1:] == [(s + t) % P for t in range(1, P)]


def test_sampled_rows_are_exact():
    """A row of Y depends on its own query and every key and value: the oracle
    on sampled query rows equals those rows of the full result."""
    n, d, heads = 30, 12, 3
    X, Wq, Wk, Wv, Wo = rand_block(n, d, heads, seed=11)
    rows = [0, 5, 17, 29]
    for causal in (False, True):
        full = A.attention_forward(X, Wq, Wk, Wv, Wo, heads, causal)
        part = A.attention_forward(X, Wq, Wk, Wv, Wo, heads, causal, rows=rows)
        np.testing.assert_array_equal(part, full[rows])


# ---------------------------------------------------------------------------
# special cases with known answers


def test_causal_first_row_is_its_own_value():
    n, d, heads = 9, 8, 2
    X, Wq, Wk, Wv, Wo = rand_block(n, d, heads, seed=13)
    Y = A.attention_forward(X, Wq, Wk, Wv, Wo, heads, True)
    np.testing.assert_allclose(Y[0], X[0] @ Wv @ Wo, rtol=1e-13, atol=1e-13)


def test_zero_queries_attend_uniformly():
    """W_q = 0: every score is 0, so each query averages the values it sees
    (all of them, or the causal prefix)."""
    n, d, heads = 10, 8, 2
    X, _, Wk, Wv, Wo = rand_block(n, d, heads, seed=15)
    Wq = np.zeros((d, d))
    V = X @ Wv
    Y = A.attention_forward(X, Wq, Wk, Wv, Wo, heads, False)
    np.testing.assert_allclose(Y, np.tile(V.mean(axis=0), (n, 1)) @ Wo, rtol=1e-13, atol=1e-13)
    Yc = A.attention_tsp(X, Wq, Wk, Wv, Wo, heads, 2, True)
    prefix = np.cumsum(V, axis=0) / np.arange(1, n + 1)[:, None]
    np.testing.assert_allclose(Yc, prefix @ Wo, rtol=1e-13, atol=1e-13)


def test_dominant_score_selects_one_value():
    """One key whose score exceeds the others by far more than the fp64
    exponent range: the softmax is one-hot and the output is that value."""
    n, dh = 6, 4
    Q = np.zeros((n, dh))
    Q[:, 0] = 1.0
    K = np.zeros((n, dh))
    K[3, 0] = 4000.0  # score 2000 for key 3, 0 for the others
    V = np.arange(n * dh, dtype=float).reshape(n, dh)
    O = A.attention_core(Q, K, V, 1)
    np.testing.assert_array_equal(O, np.tile(V[3], (n, 1)))
    O = A.attention_core_tsp(Q, K, V, 1, 3)  # the dominant key in the middle shard
    np.testing.assert_array_equal(O, np.tile(V[3], (n, 1)))
