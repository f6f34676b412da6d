"""fp64 CPU oracle for multi-head self-attention under the TSP schedule.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline legs of ``bench.py`` import this module.  The product library
never imports, loads or calls it, and it shares no code with the CUDA path.

Arithmetic: numpy float64 throughout.  Matrix products go through numpy's
matmul (a library primitive); every other step -- scaling, the mask, the
softmax, the running-max merge of key/value shards, the accumulation of the
parameter shards' partial outputs -- is written out below in the order the
definition states it.

What it computes.  Tokens X[n][d]; weights W_q, W_k, W_v [d][d] whose columns
hold the heads side by side (head h owns columns [h dh, (h+1) dh), dh =
d / n_heads) and W_o [d][d] whose rows hold the heads in the same order.

* ``attention_core`` / ``attention_forward`` -- the plain definition.
      Q = X.W_q, K = X.W_k, V = X.W_v
      O_h = softmax(Q_h K_h^T / sqrt(dh) + M) V_h        for every head h
      Y   = [O_0 | O_1 | ... ] . W_o
  M is 0, or -inf where key position > query position when ``causal``.
  Source: "Tensor Parallelism: Splitting the Math", section "Why the
  column-then-row split -- and what happens in attention": heads are
  independent, so Q, K and V are split by columns (a subset of heads per
  shard) and the output projection by rows, with one sum of the shards'
  partial outputs at the end.  The pages print neither the softmax nor its
  scale; the textbook scaled dot-product form is taken.

* ``attention_tsp`` / ``attention_core_tsp`` -- the TSP attention schedule,
  "Folding Tensor and Sequence Parallelism for Memory-Efficient Transformer
  Training & Inference", Abstract: every rank holds one sequence shard of
  tokens; the ranks iterate over the parameter shards (group w = heads
  [w H/P, (w+1) H/P)), each broadcast to all of them; with group w each
  sequence shard projects its own tokens, the shards exchange keys and values
  along the sequence so every shard's queries see the whole context, and each
  shard adds its partial output O_{s,w} . W_o[rows of group w] to its local
  accumulator.  The key/value exchange is taken as a ring: sequence shard s
  meets key/value shard (s + t) mod P at step t, and each step's scores are
  merged into a running row maximum m, row sum l and weighted sum of values
  (the standard exact merge of softmax blocks).  The result equals the plain
  definition up to rounding for any P and any visiting order.

Layout: every matrix is dense row-major, X[n][d], Y[n][d], Q/K/V/O[n][d].
"""
from __future__ import annotations

import math

import numpy as np


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # a torch tensor (any dtype): widen exactly
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _head_dim(d: int, n_heads: int) -> int:
    if n_heads <= 0 or d % n_heads:
        raise ValueError("d_model must be a multiple of n_heads")
    return d // n_heads


def _scores(q, k, q_pos, k_pos, dh, causal):
    """q[rq][dh] . k[rk][dh]^T / sqrt(dh), with -inf where a key lies after
    the query (causal)."""
    s = (q @ k.T) / math.sqrt(dh)
    if causal:
        s = np.where(k_pos[None, :] > q_pos[:, None], -np.inf, s)
    return s


def attention_core(Q, K, V, n_heads: int, causal: bool = False, rows=None):
    """Plain per-head softmax attention: O[rows][d] for queries ``rows``
    (all when None) over every key of the sequence."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    n, d = K.shape
    dh = _head_dim(d, n_heads)
    q_pos = np.arange(n) if rows is None else np.asarray(rows)
    Qr = Q
    if Qr.shape[0] != q_pos.shape[0]:
        raise ValueError("Q must have one row per query position")
    k_pos = np.arange(n)
    O = np.empty((q_pos.shape[0], d), np.float64)
    for h in range(n_heads):
        c = slice(h * dh, (h + 1) * dh)
        s = _scores(Qr[:, c], K[:, c], q_pos, k_pos, dh, causal)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        O[:, c] = (e @ V[:, c]) / e.sum(axis=1, keepdims=True)
    return O


def attention_forward(X, Wq, Wk, Wv, Wo, n_heads: int, causal: bool = False, rows=None):
    """The plain attention block: Y[rows] (all rows when None)."""
    X, Wq, Wk, Wv, Wo = map(_f64, (X, Wq, Wk, Wv, Wo))
    q_rows = X if rows is None else X[np.asarray(rows)]
    Q = q_rows @ Wq
    K = X @ Wk
    V = X @ Wv
    O = attention_core(Q, K, V, n_heads, causal, rows)
    return O @ Wo


def ring_order(s: int, t: int, P: int) -> int:
    """Key/value shard met by sequence shard s at ring step t."""
    return (s + t) % P


def reverse_ring_order(s: int, t: int, P: int) -> int:
    """The ring walked the other way round, still starting at shard s."""
    return (s - t) % P


def _merge_shards(q, K, V, q_pos, c, ns, P, s, dh, causal, order):
    """Softmax attention of the queries q (positions q_pos, columns c of one
    head) over the key/value shards visited in ``order(s, t, P)``: each
    step's scores are merged into the running maximum m, sum l and weighted
    value sum acc, rescaled by exp(m_old - m_new) whenever the maximum grows."""
    rq = q.shape[0]
    m = np.full((rq, 1), -np.inf)
    l = np.zeros((rq, 1))
    acc = np.zeros((rq, dh))
    for t in range(P):
        u = order(s, t, P)
        ku = slice(u * ns, (u + 1) * ns)
        sc = _scores(q, K[ku, c], q_pos, np.arange(u * ns, (u + 1) * ns), dh, causal)
        m_new = np.maximum(m, sc.max(axis=1, keepdims=True))
        seen = np.isfinite(m_new)  # rows with at least one visible key so far
        safe = np.where(seen, m_new, 0.0)
        scale_old = np.where(np.isfinite(m), np.exp(m - safe), 0.0)
        e = np.where(seen, np.exp(sc - safe), 0.0)
        acc = acc * scale_old + e @ V[ku, c]
        l = l * scale_old + e.sum(axis=1, keepdims=True)
        m = m_new
    return acc / l


def attention_core_tsp(Q, K, V, n_heads: int, P: int, causal: bool = False, order=ring_order):
    """The attention core under the TSP schedule: for every head, sequence
    shard s's queries meet the key/value shards in ``order`` with the running
    softmax merge.  n must be a multiple of P."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    n, d = Q.shape
    dh = _head_dim(d, n_heads)
    if P <= 0 or n % P:
        raise ValueError("n_tokens must be a multiple of P")
    ns = n // P
    O = np.empty((n, d), np.float64)
    for h in range(n_heads):
        c = slice(h * dh, (h + 1) * dh)
        for s in range(P):
            r = slice(s * ns, (s + 1) * ns)
            O[r, c] = _merge_shards(Q[r, c], K, V, np.arange(s * ns, (s + 1) * ns), c, ns, P, s,
                                    dh, causal, order)
    return O


def attention_tsp(X, Wq, Wk, Wv, Wo, n_heads: int, P: int, causal: bool = False,
                  order=ring_order, group_order=None):
    """The attention block under the TSP schedule.

    Parameter shard w = heads [w H/P, (w+1) H/P) (columns of W_q, W_k, W_v and
    rows of W_o); the shards are broadcast in ``group_order`` (0, 1, ..., P-1
    when None).  With shard w: every sequence shard projects its tokens, its
    queries meet every key/value shard in ``order``, and its partial output
    O_{s,w} . W_o[rows of w] is added to its local accumulator Y_s.  Needs
    n % P == 0 and n_heads % P == 0."""
    X, Wq, Wk, Wv, Wo = map(_f64, (X, Wq, Wk, Wv, Wo))
    n, d = X.shape
    dh = _head_dim(d, n_heads)
    if P <= 0 or n % P or n_heads % P:
        raise ValueError("n_tokens and n_heads must be multiples of P")
    ns, hw = n // P, n_heads // P
    cw = hw * dh  # columns of one parameter shard
    Y = np.zeros((n, d), np.float64)
    for w in (range(P) if group_order is None else group_order):
        cols = slice(w * cw, (w + 1) * cw)
        # every sequence shard projects its own tokens with shard w's columns
        Qw = np.empty((n, cw))
        Kw = np.empty((n, cw))
        Vw = np.empty((n, cw))
        for s in range(P):
            r = slice(s * ns, (s + 1) * ns)
            Qw[r] = X[r] @ Wq[:, cols]
            Kw[r] = X[r] @ Wk[:, cols]
            Vw[r] = X[r] @ Wv[:, cols]
        for s in range(P):
            r = slice(s * ns, (s + 1) * ns)
            Osw = np.empty((ns, cw))
            for j in range(hw):
                c = slice(j * dh, (j + 1) * dh)
                Osw[:, c] = _merge_shards(Qw[r, c], Kw, Vw, np.arange(s * ns, (s + 1) * ns), c,
                                          ns, P, s, dh, causal, order)
            Y[r] += Osw @ Wo[cols, :]
    return Y

