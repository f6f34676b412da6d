"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Nothing here touches the CUDA path.  Each pin ties the oracle to something
other than itself:

* closed forms: hand-worked 2x2 examples in ``tests/golden`` (Phi, phi and the
  logistic sigmoid, evaluated with ``math``);
* invariants the pages state: P = 1 is the unsharded block, the result does
  not depend on P or on the shard visiting order, each shard's hidden block is
  exactly the matching columns of the unsharded hidden layer, the partials sum
  to the full product ("Tensor Parallelism: Splitting the Math", steps 2-6 and
  "Why the column-then-row split"; "Folding Tensor and Sequence Parallelism
  ...", Abstract, for the ring);
* a negative test: a row-first split of A with GeLU applied to partial sums
  gives a different answer ("Why the column-then-row split");
* special cases that reduce to a library routine: GeLU in its linear and zero
  regimes, SiLU in its linear regime, where the block is a numpy matmul chain;
* derivatives: the closed-form backward against central finite differences of
  the forward and against torch autograd in fp64.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mlp_2x2_closed_form.json")


def Phi(z):
    return 0.5 * (1.0 + math.erf(z / math.sqrt(2.0)))


def phi(z):
    return math.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi)


def sig(z):
    return 1.0 / (1.0 + math.exp(-z))


def ev(expr_grid):
    ns = {"Phi": Phi, "phi": phi, "sig": sig, "__builtins__": {}}
    return np.array([[eval(e, ns) for e in row] for row in expr_grid], dtype=np.float64)


@pytest.fixture(scope="module")
def g2():
    with open(GOLDEN) as fh:
        return json.load(fh)


def _inp(g2):
    i = g2["inputs"]
    return (np.array(i["X"], float), np.array(i["A"], float), np.array(i["Wu"], float),
            np.array(i["B"], float), np.array(i["dY"], float))


def rel_fro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# ---------------------------------------------------------------------------
# closed forms


def test_golden_numbers_match_their_expressions(g2):
    for form in ("gelu", "swiglu"):
        for key, ent in g2[form].items():
            if isinstance(ent, dict) and "expr" in ent and "value" in ent:
                np.testing.assert_allclose(ev(ent["expr"]), np.array(ent["value"]), rtol=0,
                                           atol=1e-15, err_msg=f"{form}.{key}")


def test_gelu_2x2_forward(g2):
    X, A, Wu, B, _ = _inp(g2)
    Y = oracle.mlp_forward(X, A, None, B, "gelu")
    np.testing.assert_allclose(Y, ev(g2["gelu"]["Y"]["expr"]), rtol=1e-15, atol=1e-15)
    H = oracle.mlp_hidden(X, A, None, "gelu")
    np.testing.assert_allclose(H, ev(g2["gelu"]["H"]["expr"]), rtol=1e-15, atol=1e-15)


def test_gelu_2x2_shard_partials(g2):
    X, A, Wu, B, _ = _inp(g2)
    for w in (0, 1):
        Hw, Yw = oracle.mlp_shard_partial(X, A, None, B, "gelu", 2, w)
        np.testing.assert_allclose(Yw, ev(g2["gelu"][f"partial_{w}"]["expr"]), rtol=1e-15,
                                   atol=1e-15)
    Ys = oracle.mlp_sharded(X, A, None, B, "gelu", 2)
    np.testing.assert_allclose(Ys, ev(g2["gelu"]["Y"]["expr"]), rtol=1e-15, atol=1e-15)


def test_swiglu_2x2_forward(g2):
    X, A, Wu, B, _ = _inp(g2)
    Y = oracle.mlp_forward(X, A, Wu, B, "swiglu")
    np.testing.assert_allclose(Y, ev(g2["swiglu"]["Y"]["expr"]), rtol=1e-14, atol=1e-15)
    H = oracle.mlp_hidden(X, A, Wu, "swiglu")
    np.testing.assert_allclose(H, ev(g2["swiglu"]["H"]["expr"]), rtol=1e-15, atol=1e-15)
    Ys = oracle.mlp_sharded(X, A, Wu, B, "swiglu", 2, order=[1, 0])
    np.testing.assert_allclose(Ys, ev(g2["swiglu"]["Y"]["expr"]), rtol=1e-14, atol=1e-15)


def test_swiglu_2x2_backward(g2):
    X, A, Wu, B, dY = _inp(g2)
    dX, dWg, dWu, dWd = oracle.mlp_backward(X, A, Wu, B, dY, "swiglu")
    bw = g2["swiglu"]["backward_dY_identity"]
    np.testing.assert_allclose(dX, ev(bw["dX"]["expr"]), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(dWg, ev(bw["dWg"]["expr"]), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(dWu, ev(bw["dWu"]["expr"]), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(dWd, ev(bw["dWd"]["expr"]), rtol=1e-14, atol=1e-15)


def test_gelu_2x2_backward(g2):
    X, A, Wu, B, dY = _inp(g2)
    dX, dA, dWu, dB = oracle.mlp_backward(X, A, None, B, dY, "gelu")
    assert dWu is None
    bw = g2["gelu"]["backward_dY_identity"]
    np.testing.assert_allclose(dX, ev(bw["dX"]["expr"]), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(dA, ev(bw["dA"]["expr"]), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(dB, ev(bw["dB"]["expr"]), rtol=1e-14, atol=1e-15)


# ---------------------------------------------------------------------------
# the negative test: GeLU(a + b) != GeLU(a) + GeLU(b)


def _rowsplit_wrong(X, A, B, P):
    """A split by ROWS (the contraction index), GeLU applied to each rank's
    partial pre-activation, the activations summed, then .B -- the split the
    pages say is wrong.  Written with numpy and math.erf, not the oracle."""
    d = A.shape[0]
    ks = np.array_split(np.arange(d), P)
    gelu = np.vectorize(lambda z: z * Phi(z))
    H = sum(gelu(X[:, k] @ A[k, :]) for k in ks)
    return H @ B


def test_rowfirst_split_is_wrong_2x2(g2):
    X, A, Wu, B, _ = _inp(g2)
    Yw = _rowsplit_wrong(X, A, B, 2)
    np.testing.assert_allclose(Yw, ev(g2["gelu"]["Y_rowsplit_wrong"]["expr"]), rtol=1e-14)
    Y = oracle.mlp_forward(X, A, None, B, "gelu")
    assert abs(Y[0, 0] - Yw[0, 0]) > 0.2


def test_rowfirst_split_is_wrong_on_fp32_gelu_block():
    from workloads import GELU_F32, make_inputs
    t = make_inputs(GELU_F32)
    X, A, B = (t[k].double().numpy() for k in ("X", "A", "B"))
    Y = oracle.mlp_forward(X, A, None, B, "gelu")
    Yw = _rowsplit_wrong(X, A, B, GELU_F32.P)
    assert rel_fro(Yw, Y) > 1e-2
    # ... while the column-then-row split is exact
    Ys = oracle.mlp_sharded(X, A, None, B, "gelu", GELU_F32.P)
    assert rel_fro(Ys, Y) < 1e-13


# ---------------------------------------------------------------------------
# invariants of the column-then-row split and of the TSP ring


def _rand(rng, n, d, f, act, wscale=None):
    ws = wscale if wscale is not None else 1.0 / math.sqrt(d)
    X = rng.standard_normal((n, d))
    A = rng.standard_normal((d, f)) * ws
    Wu = rng.standard_normal((d, f)) * ws if act == "swiglu" else None
    B = rng.standard_normal((f, d)) / math.sqrt(f)
    return X, A, Wu, B


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_p1_is_the_unsharded_block_bitwise(act):
    rng = np.random.default_rng(11)
    X, A, Wu, B = _rand(rng, 9, 24, 40, act)
    Y = oracle.mlp_forward(X, A, Wu, B, act)
    Y1 = oracle.mlp_sharded(X, A, Wu, B, act, 1)
    assert np.array_equal(Y, Y1)


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_independent_of_P(act):
    rng = np.random.default_rng(12)
    X, A, Wu, B = _rand(rng, 13, 32, 56 * 8, act)
    Y = oracle.mlp_forward(X, A, Wu, B, act)
    for P in (1, 2, 4, 7, 8):
        YP = oracle.mlp_sharded(X, A, Wu, B, act, P)
        assert rel_fro(YP, Y) < 1e-13, P
        assert np.max(np.abs(YP - Y)) <= 1e-12 * np.max(np.abs(Y))


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_independent_of_shard_order(act):
    rng = np.random.default_rng(13)
    X, A, Wu, B = _rand(rng, 7, 16, 64, act)
    P = 8
    Y = oracle.mlp_sharded(X, A, Wu, B, act, P)
    for order in (list(range(P))[::-1], list(rng.permutation(P))):
        Yo = oracle.mlp_sharded(X, A, Wu, B, act, P, order=order)
        assert rel_fro(Yo, Y) < 1e-14


def test_bad_shard_order_is_rejected():
    rng = np.random.default_rng(14)
    X, A, Wu, B = _rand(rng, 3, 4, 8, "gelu")
    with pytest.raises(ValueError):
        oracle.mlp_sharded(X, A, None, B, "gelu", 4, order=[0, 1, 1, 2])
    with pytest.raises(ValueError):
        oracle.mlp_sharded(X, A, None, B, "gelu", 3)  # 8 % 3 != 0


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_shard_hidden_blocks_are_exact_columns_and_partials_sum(act):
    rng = np.random.default_rng(15)
    X, A, Wu, B = _rand(rng, 11, 20, 48, act)
    P = 4
    H = oracle.mlp_hidden(X, A, Wu, act)
    Y = oracle.mlp_forward(X, A, Wu, B, act)
    fs = 48 // P
    acc = np.zeros_like(Y)
    for w in range(P):
        Hw, Yw = oracle.mlp_shard_partial(X, A, Wu, B, act, P, w)
        # "GeLU(X.A1) is exactly correct locally": bitwise the same columns
        assert np.array_equal(Hw, H[:, w * fs:(w + 1) * fs])
        np.testing.assert_allclose(Yw, Hw @ B[w * fs:(w + 1) * fs, :], rtol=1e-12, atol=1e-14)
        acc += Yw
    assert rel_fro(acc, Y) < 1e-14


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_tsp_ring_equals_unsharded_and_either_direction(act):
    rng = np.random.default_rng(16)
    P = 4
    X, A, Wu, B = _rand(rng, 4 * 5, 16, 8 * P, act)
    Y = oracle.mlp_forward(X, A, Wu, B, act)
    Yt = oracle.mlp_tsp(X, A, Wu, B, act, P)
    Yr = oracle.mlp_tsp(X, A, Wu, B, act, P, reverse=True)
    assert rel_fro(Yt, Y) < 1e-14
    assert rel_fro(Yr, Y) < 1e-14
    # sequence shard 0 starts with weight shard 0, so its rows are exactly the
    # in-order sharded sum
    Ys = oracle.mlp_sharded(X, A, Wu, B, act, P)
    assert np.array_equal(Yt[:5], Ys[:5])
    # sequence shard 1 visits 1, 2, 3, 0
    Ys1 = oracle.mlp_sharded(X[5:10], A, Wu, B, act, P, order=[1, 2, 3, 0])
    assert np.array_equal(Yt[5:10], Ys1)


def test_tsp_needs_divisible_tokens():
    rng = np.random.default_rng(17)
    X, A, Wu, B = _rand(rng, 6, 4, 8, "gelu")
    with pytest.raises(ValueError):
        oracle.mlp_tsp(X, A, None, B, "gelu", 4)


# ---------------------------------------------------------------------------
# special cases that reduce to numpy matmul


def test_gelu_linear_and_zero_regimes_reduce_to_matmul():
    rng = np.random.default_rng(21)
    n, d, f = 6, 10, 12
    X = np.abs(rng.standard_normal((n, d))) + 1.0      # positive rows
    A = np.abs(rng.standard_normal((d, f))) + 1.0      # so Z = X.A >= 10
    B = rng.standard_normal((f, d))
    Z = X @ A
    assert Z.min() > 10.0  # Phi(z) = 1 to fp64 precision above z ~ 8.3
    np.testing.assert_allclose(oracle.mlp_forward(X, A, None, B, "gelu"), Z @ B, rtol=1e-13)
    Yneg = oracle.mlp_forward(X, -A, None, B, "gelu")  # Z <= -10: GeLU ~ 0
    assert np.max(np.abs(Yneg)) < 1e-15


def test_swiglu_linear_regime_reduces_to_matmul():
    rng = np.random.default_rng(22)
    n, d, f = 5, 8, 16
    X = np.abs(rng.standard_normal((n, d))) + 1.0
    Wg = np.abs(rng.standard_normal((d, f))) * 5.0 + 8.0   # G >= 64: sigmoid(G) = 1 in fp64
    Wu = rng.standard_normal((d, f))
    Wd = rng.standard_normal((f, d))
    G = X @ Wg
    assert G.min() > 40.0
    ref = ((G) * (X @ Wu)) @ Wd
    np.testing.assert_allclose(oracle.mlp_forward(X, Wg, Wu, Wd, "swiglu"), ref, rtol=1e-12,
                               atol=1e-9 * np.abs(ref).max())


# ---------------------------------------------------------------------------
# brute force: random tiny shapes against numpy + scipy special functions


@pytest.mark.parametrize("trial", range(6))
def test_brute_force_tiny_shapes(trial):
    from scipy.special import erf, expit
    rng = np.random.default_rng(100 + trial)
    n, d, f = (int(v) for v in rng.integers(1, 9, size=3))
    for act in ("gelu", "swiglu"):
        X, A, Wu, B = _rand(rng, n, d, f, act, wscale=1.0)
        Z = X @ A
        if act == "gelu":
            H = Z * 0.5 * (1.0 + erf(Z / np.sqrt(2.0)))
        else:
            H = Z * expit(Z) * (X @ Wu)
        np.testing.assert_allclose(oracle.mlp_forward(X, A, Wu, B, act), H @ B, rtol=1e-12,
                                   atol=1e-13)


# ---------------------------------------------------------------------------
# backward: central finite differences and torch autograd (fp64)


def _loss(X, A, Wu, B, dY, act):
    return float(np.sum(oracle.mlp_forward(X, A, Wu, B, act) * dY))


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_backward_central_differences(act):
    rng = np.random.default_rng(31)
    n, d, f = 4, 5, 6
    X, A, Wu, B = _rand(rng, n, d, f, act, wscale=0.7)
    dY = rng.standard_normal((n, d))
    grads = oracle.mlp_backward(X, A, Wu, B, dY, act)
    names = ("X", "A", "Wu", "B")
    h = 1e-5
    for idx, name in enumerate(names):
        if name == "Wu" and act == "gelu":
            continue
        args = [X, A, Wu, B]
        base = args[idx]
        num = np.zeros_like(base)
        for pos in np.ndindex(base.shape):
            p = base.copy()
            m = base.copy()
            p[pos] += h
            m[pos] -= h
            ap = list(args)
            am = list(args)
            ap[idx] = p
            am[idx] = m
            num[pos] = (_loss(*ap, dY, act) - _loss(*am, dY, act)) / (2 * h)
        np.testing.assert_allclose(grads[idx], num, rtol=1e-6, atol=1e-8, err_msg=name)


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_backward_matches_torch_autograd_fp64(act):
    import torch
    rng = np.random.default_rng(32)
    n, d, f = 7, 9, 16
    X, A, Wu, B = _rand(rng, n, d, f, act)
    dY = rng.standard_normal((n, d))
    tX, tA, tB = (torch.tensor(v, requires_grad=True) for v in (X, A, B))
    tWu = torch.tensor(Wu, requires_grad=True) if Wu is not None else None
    Z = tX @ tA
    if act == "gelu":
        H = torch.nn.functional.gelu(Z, approximate="none")
    else:
        H = torch.nn.functional.silu(Z) * (tX @ tWu)
    (H @ tB).backward(torch.tensor(dY))
    dX, dA, dWu, dB = oracle.mlp_backward(X, A, Wu, B, dY, act)
    np.testing.assert_allclose(dX, tX.grad.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dA, tA.grad.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dB, tB.grad.numpy(), rtol=1e-12, atol=1e-13)
    if act == "swiglu":
        np.testing.assert_allclose(dWu, tWu.grad.numpy(), rtol=1e-12, atol=1e-13)


def test_backward_on_column_subset_is_exact_for_those_columns():
    """dWg[:, J], dWu[:, J] and dWd[J, :] depend only on the columns J: the
    backward of the block restricted to J gives them exactly.  This is what
    lets parity tests sample f-columns of the weight gradients."""
    rng = np.random.default_rng(33)
    n, d, f = 6, 5, 12
    X, A, Wu, B = _rand(rng, n, d, f, "swiglu")
    dY = rng.standard_normal((n, d))
    full = oracle.mlp_backward(X, A, Wu, B, dY, "swiglu")
    J = [0, 5, 11]
    sub = oracle.mlp_backward(X, A[:, J], Wu[:, J], B[J, :], dY, "swiglu")
    assert np.array_equal(sub[1], full[1][:, J])
    assert np.array_equal(sub[2], full[2][:, J])
    assert np.array_equal(sub[3], full[3][J, :])
