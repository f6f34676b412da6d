"""Guard bands around every output buffer and the workspace.

Each output (Y, dX, the weight gradients) is a view into a larger buffer
whose margins hold a fixed bit pattern, and the workspace is followed by a
patterned tail; after the call every margin must be unchanged.  Ragged shapes
(no dimension a multiple of the tile) put partial tiles at every edge, where
an out-of-range store would land in a margin.  The values themselves are
checked against the oracle as in the parity tests.
"""
import numpy as np
import pytest
import torch

import oracle
import sequence_transformer_mlp_b200 as T
from workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

GUARD = 8192          # elements on each side (keeps views 16-byte aligned)
PATTERN16 = 0x5A5A    # bf16 margin bits
PATTERN32 = 0x5A5A5A5A


def guarded(shape, dtype):
    numel = int(np.prod(shape))
    buf = torch.empty(GUARD + numel + GUARD, dtype=dtype, device="cuda")
    if dtype == torch.bfloat16:
        buf.view(torch.int16).fill_(PATTERN16)
    else:
        buf.view(torch.int32).fill_(PATTERN32)
    return buf, buf[GUARD:GUARD + numel].view(shape)


def margins_intact(buf, numel):
    if buf.dtype == torch.bfloat16:
        bits, pat = buf.view(torch.int16), PATTERN16
    else:
        bits, pat = buf.view(torch.int32), PATTERN32
    head, tail = bits[:GUARD], bits[GUARD + numel:]
    return bool((head == pat).all()) and bool((tail == pat).all())


def guarded_workspace(nbytes):
    ws = torch.empty(nbytes + 65536, dtype=torch.uint8, device="cuda")
    ws.fill_(0xA5)
    return ws


def close(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    mx = float(np.abs(ref).max())
    assert float(np.abs(got - ref).max()) <= 1e-2 * mx, what
    assert float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)) <= 5e-3, what


@pytest.mark.parametrize("act,n,d,f,P,sched", [
    ("swiglu", 300, 200, 7 * 64, 7, "weight_shards"),
    ("gelu", 999, 264, 3 * 200, 3, "weight_shards"),
    ("swiglu", 8 * 100, 256, 8 * 128, 8, "tsp_ring"),
    ("swiglu", 8 * 100, 256, 8 * 96, 8, "tsp_ring"),
    ("swiglu", 300, 200, 7 * 64, 7, "fused"),
    ("swiglu", 300, 200, 7 * 64, 7, "shard_passes_fused"),
])
def test_forward_writes_nothing_outside_y_and_workspace(act, n, d, f, P, sched):
    wl = Workload(f"guard_{act}", act, "bf16", n, d, f, P, seed=41, w_std=0.05)
    inp = make_inputs(wl)
    dev = {k: (v.to("cuda") if v is not None else None) for k, v in inp.items()}
    ybuf, Y = guarded((n, d), torch.bfloat16)
    need = T.tsp_mlp_workspace_size(n, d, f, P, act, "bf16", sched)
    ws = guarded_workspace(need)
    T.tsp_mlp_forward_ex(dev["X"], dev["A"], dev["Wu"], dev["B"], n, d, f, P, act, "bf16", sched,
                         Y, ws, need, None)
    torch.cuda.synchronize()
    assert T.tsp_poll_device_error() == T.TSP_OK
    assert margins_intact(ybuf, n * d), "a store landed outside Y"
    assert bool((ws[need:] == 0xA5).all()), "a store landed past the workspace"
    ref = oracle.mlp_forward(inp["X"], inp["A"], inp["Wu"], inp["B"], act)
    close(Y.float().cpu().numpy(), ref, "Y")


@pytest.mark.parametrize("act,n,d,f,P", [("swiglu", 300, 200, 7 * 64, 7), ("gelu", 777, 264, 3 * 200, 3)])
def test_backward_writes_nothing_outside_its_outputs(act, n, d, f, P):
    wl = Workload(f"guard_bwd_{act}", act, "bf16", n, d, f, P, seed=42, w_std=0.05, backward=True)
    inp = make_inputs(wl)
    dev = {k: (v.to("cuda") if v is not None else None) for k, v in inp.items()}
    xbuf, dX = guarded((n, d), torch.bfloat16)
    gbuf, dWg = guarded((d, f), torch.float32)
    ubuf, dWu = guarded((d, f), torch.float32)
    dbuf, dWd = guarded((f, d), torch.float32)
    need = T.tsp_mlp_workspace_size(n, d, f, P, act, "bf16", "weight_shards", backward=True)
    ws = guarded_workspace(need)
    T.tsp_mlp_backward_ex(dev["X"], dev["A"], dev["Wu"], dev["B"], dev["dY"], n, d, f, P, act,
                          dX, dWg, dWu if act == "swiglu" else None, dWd, ws, need, None)
    torch.cuda.synchronize()
    assert T.tsp_poll_device_error() == T.TSP_OK
    assert margins_intact(xbuf, n * d), "a store landed outside dX"
    assert margins_intact(gbuf, d * f), "a store landed outside dW_gate"
    assert margins_intact(dbuf, f * d), "a store landed outside dW_down"
    if act == "swiglu":
        assert margins_intact(ubuf, d * f), "a store landed outside dW_up"
    else:
        assert margins_intact(ubuf, d * f) and bool((dWu.view(torch.int32) == PATTERN32).all()), \
            "dW_up written for the plain block"
    assert bool((ws[need:] == 0xA5).all()), "a store landed past the workspace"
    ref = oracle.mlp_backward(inp["X"], inp["A"], inp["Wu"], inp["B"], inp["dY"], act)
    close(dX.float().cpu().numpy(), ref[0], "dX")
    close(dWg.cpu().numpy(), ref[1], "dW_gate")
    close(dWd.cpu().numpy(), ref[3], "dW_down")


@pytest.mark.parametrize("act,n,d,f,P", [("gelu", 77, 45, 6 * 35, 6), ("swiglu", 700, 96, 3 * 600, 3)])
def test_fp32_forward_writes_nothing_outside_y(act, n, d, f, P):
    wl = Workload(f"guard_f32_{act}", act, "f32", n, d, f, P, seed=43, w_std=0.1)
    inp = make_inputs(wl)
    dev = {k: (v.to("cuda") if v is not None else None) for k, v in inp.items()}
    ybuf, Y = guarded((n, d), torch.float32)
    need = T.tsp_mlp_workspace_size(n, d, f, P, act, "f32")
    ws = guarded_workspace(need)
    T.tsp_mlp_forward_ex(dev["X"], dev["A"], dev["Wu"], dev["B"], n, d, f, P, act, "f32",
                         "weight_shards", Y, ws, need, None)
    torch.cuda.synchronize()
    assert T.tsp_poll_device_error() == T.TSP_OK
    assert margins_intact(ybuf, n * d), "a store landed outside Y"
    assert bool((ws[need:] == 0xA5).all()), "a store landed past the workspace"
