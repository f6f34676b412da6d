"""GPU parity of the backward pass against the fp64 oracle, through the C ABI.

Outputs: dX (bf16) and the fp32 weight gradients dW_gate (dA), dW_up and
dW_down (dB).  Each must meet the bf16 bar: max|d - ref| <= 1e-2 max|ref| and
relative Frobenius error <= 5e-3.

Small and ragged shapes are compared in full.  At the full Llama-3-8B shape
dX is compared on sampled token rows (a row of dX depends only on the same
rows of X and dY) and the weight gradients on sampled hidden columns j: the
columns j of dW_gate / dW_up and the rows j of dW_down depend only on column j
of the gate/up weights and row j of W_down, so the oracle's backward of the
block restricted to those columns gives them exactly (pinned on the CPU in
test_oracle_pins.py).
"""
import numpy as np
import pytest
import torch

import oracle
import sequence_transformer_mlp_b200 as T
from workloads import FWD_BWD, Workload, cover_cols, cover_rows, make_inputs

pytestmark = pytest.mark.gpu


def check(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, what
    assert np.isfinite(got).all(), f"{what}: non-finite"
    mx = float(np.abs(ref).max())
    err = float(np.abs(got - ref).max())
    fro = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    print(f"PARITY {what} max_rel={err / mx:.3e} fro={fro:.3e}")  # shown with pytest -s
    assert err <= 1e-2 * mx, f"{what}: max|d|/max|ref| = {err / mx:.3e}"
    assert fro <= 5e-3, f"{what}: rel Frobenius {fro:.3e}"


def np64(t):
    return t.float().cpu().double().numpy()


def gpu_backward(inp, P, act, ws_bytes=None):
    dev = {k: (v.to("cuda") if v is not None else None) for k, v in inp.items()}
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda") if ws_bytes else None
    out = T.mlp_backward(dev["X"], dev["A"], dev["Wu"], dev["B"], dev["dY"], P, act, workspace=ws)
    assert T.tsp_poll_device_error() == T.TSP_OK
    return out


CASES = [
    # degenerate: one token, d_model = 8, 8-column shards
    ("swiglu", 1, 8, 8, 1),
    ("swiglu", 3, 16, 64, 8),
    ("gelu", 257, 8, 16, 2),
    ("swiglu", 128, 64, 128, 1),
    ("swiglu", 256, 256, 512, 2),
    ("swiglu", 1000, 520, 1408, 8),
    ("swiglu", 300, 200, 7 * 64, 7),
    ("gelu", 128, 128, 256, 1),
    ("gelu", 300, 520, 1024, 4),
    ("gelu", 777, 264, 3 * 200, 3),
]


@pytest.mark.parametrize("act,n,d,f,P", CASES)
def test_backward_small_shapes(act, n, d, f, P):
    wl = Workload(f"bwd_{act}", act, "bf16", n, d, f, P, seed=n + f, w_std=0.05, backward=True)
    inp = make_inputs(wl)
    dX, dWg, dWu, dWd = gpu_backward(inp, P, act)
    ref = oracle.mlp_backward(inp["X"], inp["A"], inp["Wu"], inp["B"], inp["dY"], act)
    check(np64(dX), ref[0], "dX")
    check(np64(dWg), ref[1], "dW_gate")
    if act == "swiglu":
        check(np64(dWu), ref[2], "dW_up")
    check(np64(dWd), ref[3], "dW_down")


@pytest.mark.parametrize("act", ["swiglu", "gelu"])
def test_backward_multi_pass(act):
    """A small workspace forces 128-column chunks: dX goes through the store,
    add and final passes of its fp32 accumulator."""
    n, d, f, P = 384, 256, 4 * 256, 4
    wl = Workload("bwd_mp", act, "bf16", n, d, f, P, seed=5, w_std=0.05, backward=True)
    inp = make_inputs(wl)
    # bf16 buffers H, dG (dU) and the fp32 dH buffer of one 128-column chunk
    # each, plus the fp32 dX accumulator
    n16, n32 = (3, 1) if act == "swiglu" else (2, 1)
    ws = n * d * 4 + 2048 + n16 * (n * 128 * 2 + 256) + n32 * (n * 128 * 4 + 256) + 4096
    dX, dWg, dWu, dWd = gpu_backward(inp, P, act, ws_bytes=ws)
    ref = oracle.mlp_backward(inp["X"], inp["A"], inp["Wu"], inp["B"], inp["dY"], act)
    check(np64(dX), ref[0], "dX")
    check(np64(dWg), ref[1], "dW_gate")
    if act == "swiglu":
        check(np64(dWu), ref[2], "dW_up")
    check(np64(dWd), ref[3], "dW_down")


def test_backward_deterministic():
    wl = Workload("bwd_det", "swiglu", "bf16", 512, 256, 4 * 128, 4, seed=9, w_std=0.05,
                  backward=True)
    inp = make_inputs(wl)
    a = [np64(t) for t in gpu_backward(inp, 4, "swiglu")]
    b = [np64(t) for t in gpu_backward(inp, 4, "swiglu")]
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_tsp_mlp_backward_basic_entry_point():
    wl = Workload("bwd_basic", "swiglu", "bf16", 256, 128, 2 * 128, 2, seed=4, w_std=0.05,
                  backward=True)
    inp = make_inputs(wl)
    dev = {k: v.to("cuda") for k, v in inp.items()}
    n, d, f = 256, 128, 256
    dX = torch.empty(n, d, dtype=torch.bfloat16, device="cuda")
    g = [torch.empty(d, f, device="cuda"), torch.empty(d, f, device="cuda"),
         torch.empty(f, d, device="cuda")]
    T.tsp_mlp_backward(dev["X"], dev["A"], dev["Wu"], dev["B"], dev["dY"], n, d, f, 2, "swiglu",
                       dX, g[0], g[1], g[2])
    ref = T.mlp_backward(dev["X"], dev["A"], dev["Wu"], dev["B"], dev["dY"], 2, "swiglu")
    torch.cuda.synchronize()
    assert torch.equal(dX, ref[0])
    for a, b in zip(g, (ref[1], ref[2], ref[3])):
        assert torch.equal(a, b)


def test_fwd_bwd_llama8b_shape_sampled():
    wl = FWD_BWD
    inp = make_inputs(wl)
    dev = {k: v.to("cuda") for k, v in inp.items()}
    Y = T.mlp_forward(dev["X"], dev["A"], dev["Wu"], dev["B"], wl.P, wl.act)
    dX, dWg, dWu, dWd = T.mlp_backward(dev["X"], dev["A"], dev["Wu"], dev["B"], dev["dY"], wl.P,
                                       wl.act)
    assert T.tsp_poll_device_error() == T.TSP_OK
    # one seeded row in each of the 16 blocks of 256 token rows (every pair row
    # tile of the forward and of the input gradient), plus rows 0 and 4095
    rows = cover_rows(wl.n, 256, wl.seed)
    refY = oracle.mlp_sharded(inp["X"][rows], inp["A"], inp["Wu"], inp["B"], wl.act, wl.P)
    check(np64(Y[rows]), refY, "Y rows")
    ref_dx = oracle.mlp_backward(inp["X"][rows], inp["A"], inp["Wu"], inp["B"], inp["dY"][rows],
                                 wl.act, outputs=("dX",))[0]
    check(np64(dX[rows]), ref_dx, "dX rows")
    # hidden columns: the first and last of each of the 8 weight shards, plus one
    # seeded column in each of the 112 blocks of 128 (every 128-column tile of
    # dW_gate | dW_up, every 256-row tile of dW_down)
    cols = cover_cols(wl.f, wl.P, 128, wl.seed + 1)
    sub = oracle.mlp_backward(inp["X"], inp["A"][:, cols], inp["Wu"][:, cols], inp["B"][cols, :],
                              inp["dY"], wl.act, outputs=("dA", "dWu", "dB"))
    check(np64(dWg[:, cols]), sub[1], "dW_gate cols")
    check(np64(dWu[:, cols]), sub[2], "dW_up cols")
    check(np64(dWd[cols, :]), sub[3], "dW_down rows")
