"""fp64 CPU oracle for the column-then-row sharded transformer MLP.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` import this package.  The product library
(``sequence_transformer_mlp_b200``) never imports, loads or calls it, and it
shares no code with the CUDA path.

The arithmetic lives in ``tspmlp_oracle.c`` (plain C, fp64, OpenMP over token
rows); this module only marshals numpy arrays into it.  Which passage of the
pages each function follows is stated in the C file's header:

* ``mlp_forward``      -- the unsharded block ``Y = act(X.A).B``
  ("Tensor Parallelism: Splitting the Math", "Why the column-then-row split").
* ``mlp_hidden``       -- ``H = act(X.A)``.
* ``mlp_shard_partial`` -- one column shard's hidden block and partial output
  (same page, steps 2-5 of the two-GPU walk-through).
* ``mlp_sharded``      -- the sum of partial outputs in a given shard order
  (same page, step 6).
* ``mlp_tsp``          -- the folded tensor-and-sequence ring schedule
  ("Folding Tensor and Sequence Parallelism ...", Abstract).
* ``mlp_backward``     -- closed-form gradients of the forward definition.

Multi-head self-attention under the TSP schedule (the second runtime schedule
of "Folding Tensor and Sequence Parallelism ...", Abstract) lives in
``oracle.attention`` (numpy fp64; its header cites the passages).

Activations: ``"gelu"`` is the exact erf GeLU; ``"swiglu"`` is
``SiLU(X.Wg) * (X.Wu)``.  Matrices are row-major ``X[n,d]``, ``A=Wg[d,f]``,
``Wu[d,f]``, ``B=Wd[f,d]``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tspmlp_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

ACT = {"gelu": 0, "swiglu": 1}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-shared",
               "-fPIC", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def bind(path: str):
    """Load an oracle shared library from ``path`` and declare its signatures."""
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    i64 = ctypes.c_int64
    ci = ctypes.c_int
    lib.oracle_num_threads.restype = ci
    lib.oracle_mlp_forward.argtypes = [dp, dp, dp, dp, i64, i64, i64, ci, dp]
    lib.oracle_mlp_hidden.argtypes = [dp, dp, dp, i64, i64, i64, ci, dp]
    lib.oracle_mlp_shard_partial.argtypes = [dp, dp, dp, dp, i64, i64, i64, ci, ci, ci, dp, dp]
    lib.oracle_mlp_sharded.argtypes = [dp, dp, dp, dp, i64, i64, i64, ci, ci,
                                       ctypes.POINTER(ctypes.c_int), dp]
    lib.oracle_mlp_tsp.argtypes = [dp, dp, dp, dp, i64, i64, i64, ci, ci, ci, dp]
    lib.oracle_mlp_backward.argtypes = [dp, dp, dp, dp, dp, i64, i64, i64, ci, dp, dp, dp, dp]
    for name in ("oracle_mlp_forward", "oracle_mlp_hidden", "oracle_mlp_shard_partial",
                 "oracle_mlp_sharded", "oracle_mlp_tsp", "oracle_mlp_backward"):
        getattr(lib, name).restype = ci
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = bind(build())
    return _lib


def _f64(a):
    """A C-contiguous fp64 copy/view of ``a`` (numpy array or torch tensor)."""
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor: widen on the CPU, exactly
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name} failed with code {rc} (1 = bad arguments, 2 = out of memory)")


def _dims(X, A, Wu, B, act):
    if act not in ACT:
        raise ValueError(f"unknown activation {act!r}")
    n, d = X.shape
    d2, f = A.shape
    if d2 != d or B.shape != (f, d):
        raise ValueError("shape mismatch: need X[n,d], A[d,f], B[f,d]")
    if act == "swiglu" and (Wu is None or Wu.shape != (d, f)):
        raise ValueError("swiglu needs Wu[d,f]")
    return n, d, f


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def mlp_forward(X, A, Wu, B, act: str) -> np.ndarray:
    X, A, Wu, B = map(_f64, (X, A, Wu, B))
    n, d, f = _dims(X, A, Wu, B, act)
    Y = np.empty((n, d), np.float64)
    _check(_load().oracle_mlp_forward(_p(X), _p(A), _p(Wu), _p(B), n, d, f, ACT[act], _p(Y)),
           "oracle_mlp_forward")
    return Y


def mlp_hidden(X, A, Wu, act: str) -> np.ndarray:
    X, A, Wu = map(_f64, (X, A, Wu))
    n, d = X.shape
    f = A.shape[1]
    H = np.empty((n, f), np.float64)
    _check(_load().oracle_mlp_hidden(_p(X), _p(A), _p(Wu), n, d, f, ACT[act], _p(H)),
           "oracle_mlp_hidden")
    return H


def mlp_shard_partial(X, A, Wu, B, act: str, P: int, w: int):
    X, A, Wu, B = map(_f64, (X, A, Wu, B))
    n, d, f = _dims(X, A, Wu, B, act)
    if P <= 0 or f % P:
        raise ValueError("d_ff must be a multiple of P")
    Hw = np.empty((n, f // P), np.float64)
    Yw = np.empty((n, d), np.float64)
    _check(_load().oracle_mlp_shard_partial(_p(X), _p(A), _p(Wu), _p(B), n, d, f, ACT[act], P, w,
                                            _p(Hw), _p(Yw)), "oracle_mlp_shard_partial")
    return Hw, Yw


def mlp_sharded(X, A, Wu, B, act: str, P: int, order=None) -> np.ndarray:
    X, A, Wu, B = map(_f64, (X, A, Wu, B))
    n, d, f = _dims(X, A, Wu, B, act)
    Y = np.empty((n, d), np.float64)
    if order is None:
        optr = ctypes.POINTER(ctypes.c_int)()
    else:
        arr = (ctypes.c_int * P)(*[int(o) for o in order])
        optr = ctypes.cast(arr, ctypes.POINTER(ctypes.c_int))
    _check(_load().oracle_mlp_sharded(_p(X), _p(A), _p(Wu), _p(B), n, d, f, ACT[act], P, optr,
                                      _p(Y)), "oracle_mlp_sharded")
    return Y


def mlp_tsp(X, A, Wu, B, act: str, P: int, reverse: bool = False) -> np.ndarray:
    X, A, Wu, B = map(_f64, (X, A, Wu, B))
    n, d, f = _dims(X, A, Wu, B, act)
    Y = np.empty((n, d), np.float64)
    _check(_load().oracle_mlp_tsp(_p(X), _p(A), _p(Wu), _p(B), n, d, f, ACT[act], P,
                                  1 if reverse else 0, _p(Y)), "oracle_mlp_tsp")
    return Y


def mlp_backward(X, A, Wu, B, dY, act: str, outputs=("dX", "dA", "dWu", "dB")):
    """Returns (dX, dA, dWu, dB); dWu is None for the plain GeLU MLP, and any
    gradient not named in ``outputs`` is None (and not computed)."""
    X, A, Wu, B, dY = map(_f64, (X, A, Wu, B, dY))
    n, d, f = _dims(X, A, Wu, B, act)
    if dY.shape != (n, d):
        raise ValueError("dY must be [n,d]")
    dX = np.empty((n, d), np.float64) if "dX" in outputs else None
    dA = np.empty((d, f), np.float64) if "dA" in outputs else None
    dWu = np.empty((d, f), np.float64) if act == "swiglu" and "dWu" in outputs else None
    dB = np.empty((f, d), np.float64) if "dB" in outputs else None
    _check(_load().oracle_mlp_backward(_p(X), _p(A), _p(Wu), _p(B), _p(dY), n, d, f, ACT[act],
                                       _p(dX), _p(dA), _p(dWu), _p(dB)), "oracle_mlp_backward")
    return dX, dA, dWu, dB
