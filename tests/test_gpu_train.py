"""GPU parity of the training pair through the C ABI: tsp_mlp_forward_train
(Y and the saved activations) and tsp_mlp_backward_saved.

- Y is bit-identical to tsp_mlp_forward_ex's (the same tiles and epilogue
  arithmetic), and the saved H meets the bf16 bar against the oracle's hidden
  activations.
- dX, dW_gate and dW_up are bit-identical to tsp_mlp_backward_ex's: the saved
  factors are the recompute backward's own expressions of the same fp32 G and
  U, rounded to bf16 the same way, and dH is the same product.
- Every output meets the bf16 bar against the fp64 oracle (dW_down uses the
  forward's H, so it is compared with the oracle, not bit for bit).
"""
import numpy as np
import pytest
import torch

import oracle
import sequence_transformer_mlp_b200 as T
from workloads import FWD_BWD, Workload, cover_cols, cover_rows, make_inputs, sample_rows

pytestmark = pytest.mark.gpu


def check(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, what
    assert np.isfinite(got).all(), f"{what}: non-finite"
    mx = float(np.abs(ref).max())
    err = float(np.abs(got - ref).max())
    fro = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    print(f"PARITY {what} max_rel={err / mx:.3e} fro={fro:.3e}")
    assert err <= 1e-2 * mx, f"{what}: max|d|/max|ref| = {err / mx:.3e}"
    assert fro <= 5e-3, f"{what}: rel Frobenius {fro:.3e}"


def np64(t):
    return t.float().cpu().double().numpy()


def train_step(dev, n, d, f, P, act, ws_bytes=None):
    Y = torch.empty(n, d, dtype=torch.bfloat16, device="cuda")
    need = T.tsp_mlp_saved_size(n, d, f, P, act)
    saved = torch.empty(need, dtype=torch.uint8, device="cuda")
    T.tsp_mlp_forward_train(dev["X"], dev["A"], dev["Wu"], dev["B"], n, d, f, P, act, Y, saved,
                            need)
    dX = torch.empty(n, d, dtype=torch.bfloat16, device="cuda")
    dWg = torch.empty(d, f, device="cuda")
    dWu = torch.empty(d, f, device="cuda") if act == "swiglu" else None
    dWd = torch.empty(f, d, device="cuda")
    wsn = ws_bytes or T.tsp_mlp_backward_saved_workspace_size(n, d, f, P, act)
    ws = torch.empty(wsn, dtype=torch.uint8, device="cuda")
    T.tsp_mlp_backward_saved(dev["X"], dev["A"], dev["Wu"], dev["B"], dev["dY"], saved, need, n,
                             d, f, P, act, dX, dWg, dWu, dWd, ws, wsn)
    torch.cuda.synchronize()
    assert T.tsp_poll_device_error() == T.TSP_OK
    return Y, saved, (dX, dWg, dWu, dWd)


def saved_h(saved, n, f):
    return saved[: n * f * 2].view(torch.bfloat16).view(n, f)


CASES = [
    ("swiglu", 1, 8, 8, 1),  # degenerate: one token, d_model = 8, 8-column shards
    ("swiglu", 3, 16, 64, 8),
    ("gelu", 257, 8, 16, 2),
    ("swiglu", 128, 64, 128, 1),
    ("swiglu", 1000, 520, 1408, 8),
    ("swiglu", 300, 200, 7 * 64, 7),
    ("gelu", 300, 520, 1024, 4),
    ("gelu", 777, 264, 3 * 200, 3),
]


@pytest.mark.parametrize("act,n,d,f,P", CASES)
def test_train_pair_matches_recompute_and_oracle(act, n, d, f, P):
    wl = Workload(f"train_{act}", act, "bf16", n, d, f, P, seed=3 * n + f, w_std=0.05,
                  backward=True)
    inp = make_inputs(wl)
    dev = {k: (v.to("cuda") if v is not None else None) for k, v in inp.items()}
    Y, saved, (dX, dWg, dWu, dWd) = train_step(dev, n, d, f, P, act)
    assert torch.equal(Y, T.mlp_forward(dev["X"], dev["A"], dev["Wu"], dev["B"], P, act))
    r = T.mlp_backward(dev["X"], dev["A"], dev["Wu"], dev["B"], dev["dY"], P, act)
    torch.cuda.synchronize()
    assert torch.equal(dX, r[0]), "dX differs from the recompute backward"
    assert torch.equal(dWg, r[1]), "dW_gate differs from the recompute backward"
    if act == "swiglu":
        assert torch.equal(dWu, r[2]), "dW_up differs from the recompute backward"
    ref = oracle.mlp_backward(inp["X"], inp["A"], inp["Wu"], inp["B"], inp["dY"], act)
    check(np64(dX), ref[0], "dX")
    check(np64(dWg), ref[1], "dW_gate")
    if act == "swiglu":
        check(np64(dWu), ref[2], "dW_up")
    check(np64(dWd), ref[3], "dW_down")
    check(np64(saved_h(saved, n, f)), oracle.mlp_hidden(inp["X"], inp["A"], inp["Wu"], act),
          "saved H")


@pytest.mark.parametrize("act", ["swiglu", "gelu"])
def test_train_pair_multi_chunk(act):
    """A small workspace forces 128-column chunks of dG (dU): the dH product
    reads the factors at each chunk's columns of the saved buffer, dW_down the
    chunk's columns of the saved H, and dX goes through its fp32 accumulator."""
    n, d, f, P = 384, 256, 4 * 256, 4
    wl = Workload("train_mc", act, "bf16", n, d, f, P, seed=6, w_std=0.05, backward=True)
    inp = make_inputs(wl)
    dev = {k: (v.to("cuda") if v is not None else None) for k, v in inp.items()}
    n16 = 2 if act == "swiglu" else 1
    ws = n * d * 4 + 2048 + n16 * (n * 128 * 2 + 256) + 4096
    _, _, (dX, dWg, dWu, dWd) = train_step(dev, n, d, f, P, act, ws_bytes=ws)
    r = T.mlp_backward(dev["X"], dev["A"], dev["Wu"], dev["B"], dev["dY"], P, act)
    torch.cuda.synchronize()
    assert torch.equal(dWg, r[1])
    if act == "swiglu":
        assert torch.equal(dWu, r[2])
    ref = oracle.mlp_backward(inp["X"], inp["A"], inp["Wu"], inp["B"], inp["dY"], act)
    check(np64(dX), ref[0], "dX")
    check(np64(dWg), ref[1], "dW_gate")
    if act == "swiglu":
        check(np64(dWu), ref[2], "dW_up")
    check(np64(dWd), ref[3], "dW_down")


def test_train_pair_row_groups():
    """More token rows than one 128 MB group of H: the training forward runs
    the rows in groups on offset views of X, Y and the saved buffer."""
    n, d, f, P = 2560, 128, 8 * 3328, 8  # 2560 x 26624 x 2 B = 136 MB of H
    wl = Workload("train_rg", "swiglu", "bf16", n, d, f, P, seed=8, w_std=0.05, backward=True)
    inp = make_inputs(wl)
    dev = {k: (v.to("cuda") if v is not None else None) for k, v in inp.items()}
    Y, saved, (dX, dWg, dWu, dWd) = train_step(dev, n, d, f, P, "swiglu")
    assert torch.equal(Y, T.mlp_forward(dev["X"], dev["A"], dev["Wu"], dev["B"], P, "swiglu"))
    rows = sample_rows(n, 10, 8)
    check(np64(saved_h(saved, n, f)[rows]),
          oracle.mlp_hidden(inp["X"][rows], inp["A"], inp["Wu"], "swiglu"), "saved H rows")
    r = T.mlp_backward(dev["X"], dev["A"], dev["Wu"], dev["B"], dev["dY"], P, "swiglu")
    torch.cuda.synchronize()
    assert torch.equal(dX, r[0]) and torch.equal(dWg, r[1]) and torch.equal(dWu, r[2])


def test_train_pair_llama8b_shape():
    wl = FWD_BWD
    inp = make_inputs(wl)
    dev = {k: v.to("cuda") for k, v in inp.items()}
    n, d, f, P = wl.n, wl.d, wl.f, wl.P
    Y, saved, (dX, dWg, dWu, dWd) = train_step(dev, n, d, f, P, wl.act)
    assert torch.equal(Y, T.mlp_forward(dev["X"], dev["A"], dev["Wu"], dev["B"], P, wl.act))
    r = T.mlp_backward(dev["X"], dev["A"], dev["Wu"], dev["B"], dev["dY"], P, wl.act)
    torch.cuda.synchronize()
    assert torch.equal(dX, r[0]) and torch.equal(dWg, r[1]) and torch.equal(dWu, r[2])
    del r
    # dX, dW_gate, dW_up are bit-identical to the recompute backward (checked
    # above), whose full-shape samples are compared with the oracle in
    # test_gpu_backward.py; here they are compared with the oracle as well.
    # Hidden columns: the first and last of each of the 8 weight shards, plus
    # one seeded column in each of the 112 blocks of 128 (every 128-column tile
    # of dW_gate | dW_up, every 256-row tile of dW_down)
    cols = cover_cols(f, P, 128, wl.seed + 1)
    sub = oracle.mlp_backward(inp["X"], inp["A"][:, cols], inp["Wu"][:, cols], inp["B"][cols, :],
                              inp["dY"], wl.act, outputs=("dA", "dWu", "dB"))
    check(np64(dWg[:, cols]), sub[1], "dW_gate cols")
    check(np64(dWu[:, cols]), sub[2], "dW_up cols")
    check(np64(dWd[cols, :]), sub[3], "dW_down rows")
    # one seeded row in each of the 16 blocks of 256 token rows (every pair row
    # tile of the training forward and of the input gradient), plus rows 0, 4095
    rows = cover_rows(n, 256, wl.seed)
    ref_dx = oracle.mlp_backward(inp["X"][rows], inp["A"], inp["Wu"], inp["B"], inp["dY"][rows],
                                 wl.act, outputs=("dX",))[0]
    check(np64(dX[rows]), ref_dx, "dX rows")
    check(np64(saved_h(saved, n, f)[rows]),
          oracle.mlp_hidden(inp["X"][rows], inp["A"], inp["Wu"], wl.act), "saved H rows")


GUARD = 8192


def guarded(shape, dtype, pattern):
    numel = int(np.prod(shape))
    buf = torch.empty(GUARD + numel + GUARD, dtype=dtype, device="cuda")
    buf.view(torch.int16 if dtype == torch.bfloat16 else torch.int32).fill_(pattern)
    return buf, buf[GUARD:GUARD + numel].view(shape)


def intact(buf, numel, pattern):
    bits = buf.view(torch.int16 if buf.dtype == torch.bfloat16 else torch.int32)
    return bool((bits[:GUARD] == pattern).all()) and bool((bits[GUARD + numel:] == pattern).all())


@pytest.mark.parametrize("act,n,d,f,P", [("swiglu", 300, 200, 7 * 64, 7),
                                         ("gelu", 777, 264, 3 * 200, 3)])
def test_train_pair_writes_nothing_outside_its_buffers(act, n, d, f, P):
    wl = Workload(f"train_guard_{act}", act, "bf16", n, d, f, P, seed=44, w_std=0.05,
                  backward=True)
    inp = make_inputs(wl)
    dev = {k: (v.to("cuda") if v is not None else None) for k, v in inp.items()}
    ybuf, Y = guarded((n, d), torch.bfloat16, 0x5A5A)
    need = T.tsp_mlp_saved_size(n, d, f, P, act)
    sbuf = torch.full((need + 65536,), 0xA5, dtype=torch.uint8, device="cuda")
    T.tsp_mlp_forward_train(dev["X"], dev["A"], dev["Wu"], dev["B"], n, d, f, P, act, Y, sbuf,
                            need)
    torch.cuda.synchronize()
    assert T.tsp_poll_device_error() == T.TSP_OK
    assert intact(ybuf, n * d, 0x5A5A), "a store landed outside Y"
    assert bool((sbuf[need:] == 0xA5).all()), "a store landed past the saved buffer"
    xbuf, dX = guarded((n, d), torch.bfloat16, 0x5A5A)
    gbuf, dWg = guarded((d, f), torch.float32, 0x5A5A5A5A)
    ubuf, dWu = guarded((d, f), torch.float32, 0x5A5A5A5A)
    dbuf, dWd = guarded((f, d), torch.float32, 0x5A5A5A5A)
    wsn = T.tsp_mlp_backward_saved_workspace_size(n, d, f, P, act)
    ws = torch.full((wsn + 65536,), 0xA5, dtype=torch.uint8, device="cuda")
    saved_copy = sbuf.clone()
    T.tsp_mlp_backward_saved(dev["X"], dev["A"], dev["Wu"], dev["B"], dev["dY"], sbuf, need, n, d,
                             f, P, act, dX, dWg, dWu if act == "swiglu" else None, dWd, ws, wsn)
    torch.cuda.synchronize()
    assert T.tsp_poll_device_error() == T.TSP_OK
    assert torch.equal(sbuf, saved_copy), "the backward wrote into the saved buffer"
    assert intact(xbuf, n * d, 0x5A5A), "a store landed outside dX"
    assert intact(gbuf, d * f, 0x5A5A5A5A), "a store landed outside dW_gate"
    assert intact(dbuf, f * d, 0x5A5A5A5A), "a store landed outside dW_down"
    if act == "swiglu":
        assert intact(ubuf, d * f, 0x5A5A5A5A), "a store landed outside dW_up"
    else:
        assert bool((dWu.view(torch.int32) == 0x5A5A5A5A).all()), "dW_up written for GeLU"
    assert bool((ws[wsn:] == 0xA5).all()), "a store landed past the workspace"
    ref = oracle.mlp_backward(inp["X"], inp["A"], inp["Wu"], inp["B"], inp["dY"], act)
    check(np64(dX), ref[0], "dX")
    check(np64(dWd), ref[3], "dW_down")


def test_torch_conveniences_match_the_entry_points():
    n, d, f, P, act = 260, 128, 4 * 128, 4, "swiglu"
    wl = Workload("train_conv", act, "bf16", n, d, f, P, seed=12, w_std=0.05, backward=True)
    inp = make_inputs(wl)
    dev = {k: (v.to("cuda") if v is not None else None) for k, v in inp.items()}
    Y, saved, g = train_step(dev, n, d, f, P, act)
    Y2, saved2 = T.mlp_forward_train(dev["X"], dev["A"], dev["Wu"], dev["B"], P, act)
    g2 = T.mlp_backward_saved(dev["X"], dev["A"], dev["Wu"], dev["B"], dev["dY"], saved2, P, act)
    torch.cuda.synchronize()
    assert T.tsp_poll_device_error() == T.TSP_OK
    assert torch.equal(Y, Y2)
    for a, b in zip(g, g2):
        assert torch.equal(a, b)
