"""Python binding of libtspmlp, the column-then-row sharded transformer MLP on
one B200 (sm_100a).

Argument marshalling only: every function below forwards to the C entry
point of the same name in ``libtspmlp.so`` (declared in ``include/tspmlp.h``),
and every step of the computation runs in the library's CUDA kernels.  There
is no CPU fallback: if the library is missing, importing a function raises.
PyTorch is used only for device memory and streams (``mlp_forward`` and
``mlp_backward`` allocate outputs and workspace with it).

Arguments that are device buffers accept a ``torch.Tensor`` (its
``data_ptr()`` is passed) or a plain integer address.  ``stream`` defaults to
the current torch CUDA stream.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtspmlp.so")

TSP_OK = 0
TSP_ERR_TIMEOUT = 5
STATUS_NAMES = {
    0: "TSP_OK",
    1: "TSP_ERR_INVALID_ARG",
    2: "TSP_ERR_UNSUPPORTED_SHAPE",
    3: "TSP_ERR_ARCH",
    4: "TSP_ERR_CUDA",
    5: "TSP_ERR_TIMEOUT",
    6: "TSP_ERR_WORKSPACE",
    7: "TSP_ERR_SCRATCH_LIMIT",
    8: "TSP_ERR_RANGE",
}
NOALLOC_SCRATCH_BYTES = 32 << 20
ACT = {"gelu": 0, "swiglu": 1}
DTYPE = {"bf16": 0, "f32": 1}
SCHED = {"weight_shards": 0, "tsp_ring": 1, "shard_passes": 2, "fused": 3,
         "tsp_ring_fused": 4, "shard_passes_fused": 5}


class KernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_int64),
                ("total_ms", ctypes.c_double)]


class TspError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load libtspmlp.so (built by ``python -m sequence_transformer_mlp_b200.build``)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"libtspmlp.so not found at {p}; build it with "
                          "`python -m sequence_transformer_mlp_b200.build`")
    lib = ctypes.CDLL(p)
    vp, i64, ci, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    lib.tsp_mlp_forward.argtypes = [vp, vp, vp, vp, i64, i64, i64, ci, ci, vp, vp]
    lib.tsp_mlp_forward_ex.argtypes = [vp, vp, vp, vp, i64, i64, i64, ci, ci, ci, ci, vp, vp, sz,
                                       vp]
    lib.tsp_mlp_forward_noalloc.argtypes = [vp, vp, vp, vp, i64, i64, i64, ci, ci, vp, vp]
    lib.tsp_mlp_backward.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, ci, ci, vp, vp, vp, vp,
                                     vp]
    lib.tsp_mlp_backward_ex.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, ci, ci, vp, vp, vp,
                                        vp, vp, sz, vp]
    lib.tsp_mlp_workspace_size.argtypes = [i64, i64, i64, ci, ci, ci, ci, ci,
                                           ctypes.POINTER(ctypes.c_size_t)]
    lib.tsp_mlp_saved_size.argtypes = [i64, i64, i64, ci, ci, ctypes.POINTER(ctypes.c_size_t)]
    lib.tsp_mlp_forward_train.argtypes = [vp, vp, vp, vp, i64, i64, i64, ci, ci, vp, vp, sz, vp]
    lib.tsp_mlp_backward_saved_workspace_size.argtypes = [i64, i64, i64, ci, ci,
                                                          ctypes.POINTER(ctypes.c_size_t)]
    lib.tsp_mlp_backward_saved.argtypes = [vp, vp, vp, vp, vp, vp, sz, i64, i64, i64, ci, ci, vp,
                                           vp, vp, vp, vp, sz, vp]
    lib.tsp_attn_core.argtypes = [vp, vp, vp, i64, i64, ci, ci, ci, vp, vp]
    lib.tsp_attn_workspace_size.argtypes = [i64, i64, ci, ci, ctypes.POINTER(ctypes.c_size_t)]
    lib.tsp_attn_forward.argtypes = [vp, vp, vp, vp, vp, i64, i64, ci, ci, ci, vp, vp, sz, vp]
    lib.tsp_status_string.argtypes = [ci]
    lib.tsp_status_string.restype = ctypes.c_char_p
    lib.tsp_poll_device_error.argtypes = [vp]
    lib.tsp_selftest_timeout.argtypes = [ci, vp]
    lib.tsp_trace_enable.argtypes = [ci]
    lib.tsp_trace_collect.argtypes = [ctypes.POINTER(KernelStat), ci, ctypes.POINTER(ci)]
    lib.tsp_trace_reset.argtypes = []
    for name in ("tsp_mlp_forward", "tsp_mlp_forward_ex", "tsp_mlp_forward_noalloc",
                 "tsp_mlp_backward",
                 "tsp_mlp_backward_ex", "tsp_mlp_workspace_size", "tsp_poll_device_error",
                 "tsp_trace_enable", "tsp_trace_collect", "tsp_trace_reset",
                 "tsp_selftest_timeout", "tsp_mlp_saved_size", "tsp_mlp_forward_train",
                 "tsp_mlp_backward_saved_workspace_size", "tsp_mlp_backward_saved",
                 "tsp_attn_core", "tsp_attn_workspace_size", "tsp_attn_forward"):
        getattr(lib, name).restype = ci
    if path is None:
        _lib = lib
    return lib


def _addr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _enum(table, v):
    return table[v] if isinstance(v, str) else int(v)


def _check(status: int, where: str) -> None:
    if status != TSP_OK:
        raise TspError(status, where)


# --------------------------------------------------------------------------- C entry points


def tsp_mlp_forward(X, W_gate, W_up, W_down, n_tokens, d_model, d_ff, P, act, Y, stream=None,
                    check=True) -> int:
    s = load().tsp_mlp_forward(_addr(X), _addr(W_gate), _addr(W_up), _addr(W_down), n_tokens,
                               d_model, d_ff, P, _enum(ACT, act), _addr(Y), _stream(stream))
    if check:
        _check(s, "tsp_mlp_forward")
    return s


def tsp_mlp_forward_ex(X, W_gate, W_up, W_down, n_tokens, d_model, d_ff, P, act, dtype, sched, Y,
                       workspace, workspace_bytes, stream=None, check=True) -> int:
    s = load().tsp_mlp_forward_ex(_addr(X), _addr(W_gate), _addr(W_up), _addr(W_down), n_tokens,
                                  d_model, d_ff, P, _enum(ACT, act), _enum(DTYPE, dtype),
                                  _enum(SCHED, sched), _addr(Y), _addr(workspace),
                                  workspace_bytes, _stream(stream))
    if check:
        _check(s, "tsp_mlp_forward_ex")
    return s


def tsp_mlp_forward_noalloc(X, W_gate, W_up, W_down, n_tokens, d_model, d_ff, P, act, Y,
                            stream=None, check=True) -> int:
    """The forward pass without any allocation: its scratch is a static device
    array of NOALLOC_SCRATCH_BYTES inside the library (see include/tspmlp.h)."""
    s = load().tsp_mlp_forward_noalloc(_addr(X), _addr(W_gate), _addr(W_up), _addr(W_down),
                                       n_tokens, d_model, d_ff, P, _enum(ACT, act), _addr(Y),
                                       _stream(stream))
    if check:
        _check(s, "tsp_mlp_forward_noalloc")
    return s


def tsp_mlp_backward(X, W_gate, W_up, W_down, dY, n_tokens, d_model, d_ff, P, act, dX, dW_gate,
                     dW_up, dW_down, stream=None, check=True) -> int:
    s = load().tsp_mlp_backward(_addr(X), _addr(W_gate), _addr(W_up), _addr(W_down), _addr(dY),
                                n_tokens, d_model, d_ff, P, _enum(ACT, act), _addr(dX),
                                _addr(dW_gate), _addr(dW_up), _addr(dW_down), _stream(stream))
    if check:
        _check(s, "tsp_mlp_backward")
    return s


def tsp_mlp_backward_ex(X, W_gate, W_up, W_down, dY, n_tokens, d_model, d_ff, P, act, dX, dW_gate,
                        dW_up, dW_down, workspace, workspace_bytes, stream=None,
                        check=True) -> int:
    s = load().tsp_mlp_backward_ex(_addr(X), _addr(W_gate), _addr(W_up), _addr(W_down),
                                   _addr(dY), n_tokens, d_model, d_ff, P, _enum(ACT, act),
                                   _addr(dX), _addr(dW_gate), _addr(dW_up), _addr(dW_down),
                                   _addr(workspace), workspace_bytes, _stream(stream))
    if check:
        _check(s, "tsp_mlp_backward_ex")
    return s


def tsp_mlp_workspace_size(n_tokens, d_model, d_ff, P, act, dtype="bf16", sched="weight_shards",
                           backward=False) -> int:
    out = ctypes.c_size_t(0)
    s = load().tsp_mlp_workspace_size(n_tokens, d_model, d_ff, P, _enum(ACT, act),
                                      _enum(DTYPE, dtype), _enum(SCHED, sched),
                                      1 if backward else 0, ctypes.byref(out))
    _check(s, "tsp_mlp_workspace_size")
    return int(out.value)


def tsp_mlp_saved_size(n_tokens, d_model, d_ff, P, act) -> int:
    out = ctypes.c_size_t(0)
    s = load().tsp_mlp_saved_size(n_tokens, d_model, d_ff, P, _enum(ACT, act), ctypes.byref(out))
    _check(s, "tsp_mlp_saved_size")
    return int(out.value)


def tsp_mlp_forward_train(X, W_gate, W_up, W_down, n_tokens, d_model, d_ff, P, act, Y, saved,
                          saved_bytes, stream=None, check=True) -> int:
    s = load().tsp_mlp_forward_train(_addr(X), _addr(W_gate), _addr(W_up), _addr(W_down),
                                     n_tokens, d_model, d_ff, P, _enum(ACT, act), _addr(Y),
                                     _addr(saved), saved_bytes, _stream(stream))
    if check:
        _check(s, "tsp_mlp_forward_train")
    return s


def tsp_mlp_backward_saved_workspace_size(n_tokens, d_model, d_ff, P, act) -> int:
    out = ctypes.c_size_t(0)
    s = load().tsp_mlp_backward_saved_workspace_size(n_tokens, d_model, d_ff, P, _enum(ACT, act),
                                                     ctypes.byref(out))
    _check(s, "tsp_mlp_backward_saved_workspace_size")
    return int(out.value)


def tsp_mlp_backward_saved(X, W_gate, W_up, W_down, dY, saved, saved_bytes, n_tokens, d_model,
                           d_ff, P, act, dX, dW_gate, dW_up, dW_down, workspace, workspace_bytes,
                           stream=None, check=True) -> int:
    s = load().tsp_mlp_backward_saved(_addr(X), _addr(W_gate), _addr(W_up), _addr(W_down),
                                      _addr(dY), _addr(saved), saved_bytes, n_tokens, d_model,
                                      d_ff, P, _enum(ACT, act), _addr(dX), _addr(dW_gate),
                                      _addr(dW_up), _addr(dW_down), _addr(workspace),
                                      workspace_bytes, _stream(stream))
    if check:
        _check(s, "tsp_mlp_backward_saved")
    return s


def tsp_attn_core(Q, K, V, n_tokens, d_model, n_heads, P, causal, O, stream=None,
                  check=True) -> int:
    s = load().tsp_attn_core(_addr(Q), _addr(K), _addr(V), n_tokens, d_model, n_heads, P,
                             1 if causal else 0, _addr(O), _stream(stream))
    if check:
        _check(s, "tsp_attn_core")
    return s


def tsp_attn_workspace_size(n_tokens, d_model, n_heads, P) -> int:
    out = ctypes.c_size_t(0)
    s = load().tsp_attn_workspace_size(n_tokens, d_model, n_heads, P, ctypes.byref(out))
    _check(s, "tsp_attn_workspace_size")
    return int(out.value)


def tsp_attn_forward(X, W_q, W_k, W_v, W_o, n_tokens, d_model, n_heads, P, causal, Y, workspace,
                     workspace_bytes, stream=None, check=True) -> int:
    s = load().tsp_attn_forward(_addr(X), _addr(W_q), _addr(W_k), _addr(W_v), _addr(W_o),
                                n_tokens, d_model, n_heads, P, 1 if causal else 0, _addr(Y),
                                _addr(workspace), workspace_bytes, _stream(stream))
    if check:
        _check(s, "tsp_attn_forward")
    return s


def tsp_status_string(status: int) -> str:
    return load().tsp_status_string(int(status)).decode()


def tsp_poll_device_error(stream=None) -> int:
    return int(load().tsp_poll_device_error(_stream(stream)))


def tsp_selftest_timeout(mode: int, stream=None) -> None:
    """Launch the failure-detection self-test (see include/tspmlp.h); the next
    tsp_poll_device_error() is expected to return TSP_ERR_TIMEOUT."""
    _check(load().tsp_selftest_timeout(int(mode), _stream(stream)), "tsp_selftest_timeout")


def tsp_trace_enable(enable: bool = True) -> None:
    _check(load().tsp_trace_enable(1 if enable else 0), "tsp_trace_enable")


def tsp_trace_collect(capacity: int = 64) -> dict:
    """{kernel name: (launches, total_ms)} accumulated since the last reset."""
    arr = (KernelStat * capacity)()
    cnt = ctypes.c_int(0)
    _check(load().tsp_trace_collect(arr, capacity, ctypes.byref(cnt)), "tsp_trace_collect")
    return {arr[i].name.decode(): (int(arr[i].launches), float(arr[i].total_ms))
            for i in range(cnt.value)}


def tsp_trace_reset() -> None:
    _check(load().tsp_trace_reset(), "tsp_trace_reset")


# --------------------------------------------------------------------------- torch conveniences


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def mlp_forward(X, W_gate, W_up, W_down, P: int, act: str, sched: str = "weight_shards",
                out=None, workspace=None, stream=None):
    """Y = act-MLP(X) through tsp_mlp_forward_ex; dtype follows X (bf16 or fp32).
    Allocates Y and the preferred workspace with torch unless given; a given
    workspace tensor is passed with its own size (the schedule adapts to it)."""
    import torch
    n, d = X.shape
    f = W_gate.shape[1]
    dt = "bf16" if X.dtype == torch.bfloat16 else "f32"
    Y = out if out is not None else torch.empty((n, d), dtype=X.dtype, device=X.device)
    if workspace is None:
        need = tsp_mlp_workspace_size(n, d, f, P, act, dt, sched)
        ws = torch.empty(need, dtype=torch.uint8, device=X.device) if need else None
    else:
        ws, need = workspace, _nbytes(workspace)
    tsp_mlp_forward_ex(X, W_gate, W_up, W_down, n, d, f, P, act, dt, sched, Y, ws, need, stream)
    return Y


def mlp_backward(X, W_gate, W_up, W_down, dY, P: int, act: str, workspace=None, stream=None):
    """(dX bf16, dW_gate fp32, dW_up fp32 or None, dW_down fp32) through
    tsp_mlp_backward_ex; a given workspace tensor is passed with its own size."""
    import torch
    n, d = X.shape
    f = W_gate.shape[1]
    dev = X.device
    dX = torch.empty((n, d), dtype=torch.bfloat16, device=dev)
    dWg = torch.empty((d, f), dtype=torch.float32, device=dev)
    dWu = torch.empty((d, f), dtype=torch.float32, device=dev) if act == "swiglu" else None
    dWd = torch.empty((f, d), dtype=torch.float32, device=dev)
    if workspace is None:
        need = tsp_mlp_workspace_size(n, d, f, P, act, "bf16", "weight_shards", backward=True)
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
    else:
        ws, need = workspace, _nbytes(workspace)
    tsp_mlp_backward_ex(X, W_gate, W_up, W_down, dY, n, d, f, P, act, dX, dWg, dWu, dWd, ws, need,
                        stream)
    return dX, dWg, dWu, dWd


def mlp_forward_train(X, W_gate, W_up, W_down, P: int, act: str, stream=None):
    """(Y, saved) through tsp_mlp_forward_train (bf16): Y as mlp_forward gives
    it, and the uint8 buffer of activations that mlp_backward_saved reads."""
    import torch
    n, d = X.shape
    f = W_gate.shape[1]
    Y = torch.empty((n, d), dtype=torch.bfloat16, device=X.device)
    need = tsp_mlp_saved_size(n, d, f, P, act)
    saved = torch.empty(need, dtype=torch.uint8, device=X.device)
    tsp_mlp_forward_train(X, W_gate, W_up, W_down, n, d, f, P, act, Y, saved, need, stream)
    return Y, saved


def mlp_backward_saved(X, W_gate, W_up, W_down, dY, saved, P: int, act: str, workspace=None,
                       stream=None):
    """(dX bf16, dW_gate fp32, dW_up fp32 or None, dW_down fp32) through
    tsp_mlp_backward_saved, from the buffer mlp_forward_train returned for the
    same X and weights; a given workspace tensor is passed with its own size."""
    import torch
    n, d = X.shape
    f = W_gate.shape[1]
    dev = X.device
    dX = torch.empty((n, d), dtype=torch.bfloat16, device=dev)
    dWg = torch.empty((d, f), dtype=torch.float32, device=dev)
    dWu = torch.empty((d, f), dtype=torch.float32, device=dev) if act == "swiglu" else None
    dWd = torch.empty((f, d), dtype=torch.float32, device=dev)
    if workspace is None:
        need = tsp_mlp_backward_saved_workspace_size(n, d, f, P, act)
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
    else:
        ws, need = workspace, _nbytes(workspace)
    tsp_mlp_backward_saved(X, W_gate, W_up, W_down, dY, saved, _nbytes(saved), n, d, f, P, act, dX,
                           dWg, dWu, dWd, ws, need, stream)
    return dX, dWg, dWu, dWd


def attn_core(Q, K, V, n_heads: int, P: int, causal: bool, out=None, stream=None):
    """O = attention(Q, K, V) through tsp_attn_core (bf16 [n, d] each)."""
    import torch
    n, d = Q.shape
    O = out if out is not None else torch.empty((n, d), dtype=torch.bfloat16, device=Q.device)
    tsp_attn_core(Q, K, V, n, d, n_heads, P, causal, O, stream)
    return O


def attn_forward(X, W_q, W_k, W_v, W_o, n_heads: int, P: int, causal: bool, workspace=None,
                 out=None, stream=None):
    """Y = attention block (X) under the TSP schedule through tsp_attn_forward;
    allocates Y and the workspace with torch unless given."""
    import torch
    n, d = X.shape
    Y = out if out is not None else torch.empty((n, d), dtype=torch.bfloat16, device=X.device)
    need = tsp_attn_workspace_size(n, d, n_heads, P)
    ws = workspace if workspace is not None else torch.empty(need, dtype=torch.uint8,
                                                              device=X.device)
    tsp_attn_forward(X, W_q, W_k, W_v, W_o, n, d, n_heads, P, causal, Y, ws, _nbytes(ws), stream)
    return Y
