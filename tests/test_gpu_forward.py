"""GPU parity of the forward pass against the fp64 oracle, through the C ABI.

Tolerances: bf16 inputs with fp32 accumulation need max|Y - Yref| <=
1e-2 max|Yref| and relative Frobenius error <= 5e-3; the fp32 path needs both
within 1e-5.  The oracle sees the exact bf16 (or fp32) input values widened to
fp64, so input quantisation is not counted as error.

Small and ragged shapes are compared element by element in full (several
tiles and a ragged tail in every dimension); the full-size workloads are
compared on sampled token rows, which the oracle computes exactly because a
row of Y depends only on the same row of X.
"""
import numpy as np
import pytest
import torch

import oracle
import sequence_transformer_mlp_b200 as T
from workloads import (GELU_F32, LLAMA8B, LLAMA70B, TSP_RING, Workload, cover_rows, make_inputs,
                       sample_rows)

pytestmark = pytest.mark.gpu


def check(got, ref, dtype, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    mx = float(np.abs(ref).max())
    err = float(np.abs(got - ref).max())
    fro = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    print(f"PARITY {what} max_rel={err / mx:.3e} fro={fro:.3e}")  # shown with pytest -s
    if dtype == "f32":
        assert err <= 1e-5 * mx and fro <= 1e-5, f"{what}: max {err / mx:.3e} fro {fro:.3e}"
    else:
        assert err <= 1e-2 * mx, f"{what}: max|d|/max|ref| = {err / mx:.3e}"
        assert fro <= 5e-3, f"{what}: rel Frobenius {fro:.3e}"
    return err / mx, fro


def to_dev(t):
    return None if t is None else t.to("cuda", non_blocking=False)


def gpu_forward(inp, P, act, sched="weight_shards", ws_bytes=None):
    X, A, Wu, B = (to_dev(inp[k]) for k in ("X", "A", "Wu", "B"))
    ws = None
    if ws_bytes is not None:
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    Y = T.mlp_forward(X, A, Wu, B, P, act, sched=sched, workspace=ws)
    assert T.tsp_poll_device_error() == T.TSP_OK
    return Y.float().cpu().double().numpy()


def small(act, dtype, n, d, f, P, seed, w_std=0.05):
    return Workload(f"{act}_{dtype}_{n}x{d}x{f}_P{P}", act, dtype, n, d, f, P, seed, w_std)


# ---------------------------------------------------------------------------- fp32 path


def test_gelu_fp32_block_exact_config():
    """The fp32 GeLU block: n=64, d_model=128, d_ff=512, P=2, seed 0."""
    inp = make_inputs(GELU_F32)
    Y = gpu_forward(inp, GELU_F32.P, "gelu")
    ref = oracle.mlp_forward(inp["X"], inp["A"], None, inp["B"], "gelu")
    check(Y, ref, "f32", "gelu fp32 P=2")
    refs = oracle.mlp_sharded(inp["X"], inp["A"], None, inp["B"], "gelu", GELU_F32.P)
    check(Y, refs, "f32", "vs sharded oracle")


@pytest.mark.parametrize("P", [1, 2, 4, 8])
@pytest.mark.parametrize("sched", ["weight_shards", "tsp_ring"])
def test_gelu_fp32_any_P_and_schedule(P, sched):
    inp = make_inputs(GELU_F32)
    Y = gpu_forward(inp, P, "gelu", sched)
    ref = oracle.mlp_forward(inp["X"], inp["A"], None, inp["B"], "gelu")
    check(Y, ref, "f32", f"P={P} {sched}")


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_fp32_large_tiles(act):
    """Enough hidden tiles for the 64 x 64 fp32 tiles (the down projection,
    with fewer, takes the 16 x 16 ones); ragged in every dimension."""
    wl = small(act, "f32", 700, 96, 3 * 600, 3, seed=6, w_std=0.1)
    inp = make_inputs(wl)
    Y = gpu_forward(inp, wl.P, act)
    ref = oracle.mlp_forward(inp["X"], inp["A"], inp["Wu"], inp["B"], act)
    check(Y, ref, "f32", wl.name)


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_fp32_ragged(act):
    wl = small(act, "f32", 77, 45, 6 * 35, 6, seed=5, w_std=0.1)
    inp = make_inputs(wl)
    Y = gpu_forward(inp, wl.P, act)
    ref = oracle.mlp_forward(inp["X"], inp["A"], inp["Wu"], inp["B"], act)
    check(Y, ref, "f32", wl.name)


# ---------------------------------------------------------------------------- bf16 tensor cores

BF16_CASES = [
    # act, n, d, f, P  -- one tile; multi-tile; ragged everywhere; odd P
    ("swiglu", 128, 64, 128, 1),
    ("swiglu", 256, 256, 512, 2),
    ("swiglu", 1000, 520, 1408, 8),
    ("swiglu", 300, 200, 7 * 64, 7),
    ("swiglu", 64, 4096, 8 * 128, 8),
    ("gelu", 128, 128, 256, 1),
    ("gelu", 300, 520, 1024, 4),
    ("gelu", 999, 264, 3 * 200, 3),
]


# Degenerate shapes: one token, the narrowest rows TMA takes (d_model = 8),
# 8-column shards, odd P -- every tile mostly zero-filled padding.
DEGENERATE_CASES = [
    ("swiglu", 1, 8, 8, 1),
    ("swiglu", 3, 16, 64, 8),
    ("gelu", 257, 8, 16, 2),
    ("swiglu", 513, 24, 40, 5),
]


@pytest.mark.parametrize("act,n,d,f,P", DEGENERATE_CASES)
def test_bf16_degenerate_shapes(act, n, d, f, P):
    wl = small(act, "bf16", n, d, f, P, seed=31)
    inp = make_inputs(wl)
    Y = gpu_forward(inp, P, act)
    ref = oracle.mlp_forward(inp["X"], inp["A"], inp["Wu"], inp["B"], act)
    check(Y, ref, "bf16", wl.name)


@pytest.mark.parametrize("n,d,f,P", [(8, 8, 8 * 8, 8), (16, 16, 2 * 64, 2)])
def test_bf16_tsp_ring_degenerate(n, d, f, P):
    """One-token and eight-token sequence shards (per-step ring passes with
    8-column shards; rotated passes with 64-column shards)."""
    wl = small("swiglu", "bf16", n, d, f, P, seed=32)
    inp = make_inputs(wl)
    Y = gpu_forward(inp, P, "swiglu", "tsp_ring")
    ref = oracle.mlp_tsp(inp["X"], inp["A"], inp["Wu"], inp["B"], "swiglu", P)
    check(Y, ref, "bf16", "tsp ring degenerate")


@pytest.mark.parametrize("act,n,d,f,P", [("gelu", 1, 1, 1, 1), ("swiglu", 5, 3, 6, 3)])
def test_fp32_degenerate_shapes(act, n, d, f, P):
    wl = small(act, "f32", n, d, f, P, seed=33, w_std=0.3)
    inp = make_inputs(wl)
    Y = gpu_forward(inp, P, act)
    ref = oracle.mlp_forward(inp["X"], inp["A"], inp["Wu"], inp["B"], act)
    check(Y, ref, "f32", wl.name)


@pytest.mark.parametrize("sched", ["weight_shards", "shard_passes_fused", "fused"])
@pytest.mark.parametrize("act,n,d,f,P", BF16_CASES)
def test_bf16_small_shapes(act, n, d, f, P, sched):
    if sched == "shard_passes_fused" and (f // P) % 64:
        pytest.skip("the one-launch passes need 64-multiple shards")
    wl = small(act, "bf16", n, d, f, P, seed=n + d + f + P)
    inp = make_inputs(wl)
    Y = gpu_forward(inp, P, act, sched)
    ref = oracle.mlp_forward(inp["X"], inp["A"], inp["Wu"], inp["B"], act)
    check(Y, ref, "bf16", wl.name)


@pytest.mark.parametrize("act", ["swiglu", "gelu"])
def test_bf16_multi_pass_accumulation(act):
    """The pass schedule with a workspace below its preferred size uses narrow
    hidden chunks, so the fp32 accumulator goes through store, add and final
    passes."""
    n, d, f, P = 384, 256, 8 * 192, 8
    wl = small(act, "bf16", n, d, f, P, seed=77)
    inp = make_inputs(wl)
    ws = n * d * 4 + 256 + n * 2 * 128 + 512   # one 128-column chunk + accumulator
    Y = gpu_forward(inp, P, act, "shard_passes", ws_bytes=ws)
    ref = oracle.mlp_forward(inp["X"], inp["A"], inp["Wu"], inp["B"], act)
    check(Y, ref, "bf16", "multi-pass")
    Y2 = gpu_forward(inp, P, act)  # the fused schedule agrees closely
    assert np.abs(Y2 - Y).max() <= 2e-2 * np.abs(ref).max()


def _a256(b):
    return (b + 255) // 256 * 256


@pytest.mark.parametrize("act", ["swiglu", "gelu"])
def test_bf16_one_launch_passes_many_chunks(act):
    """The chunked passes in one paired launch; a small workspace forces 8
    chunks, so the fp32 accumulator goes through store, add and final, and the
    two H chunk buffers are reused."""
    n, d, f, P = 4 * 256 - 37, 320, 8 * 128, 8
    wl = small(act, "bf16", n, d, f, P, seed=79)
    inp = make_inputs(wl)
    mp = (n + 255) // 256
    ws = _a256(n * d * 4) + _a256((1 + 2 * 32 * mp) * 4) + 512 + 2 * _a256(n * 128 * 2) + 256
    Y = gpu_forward(inp, P, act, "shard_passes_fused", ws_bytes=ws)
    ref = oracle.mlp_forward(inp["X"], inp["A"], inp["Wu"], inp["B"], act)
    check(Y, ref, "bf16", "one-launch passes, 8 chunks")


@pytest.mark.parametrize("act", ["swiglu", "gelu"])
def test_bf16_fused_small_ring_reuses_slots(act):
    """A workspace with room for only three H-ring slots (groups of one row
    block): every gate/up tile past the third row block waits for the down
    tiles of the row block three earlier before overwriting its slot."""
    n, d, f, P = 16 * 128 - 40, 256, 4 * 320, 4
    wl = small(act, "bf16", n, d, f, P, seed=78)
    inp = make_inputs(wl)
    slot = 128 * f * 2
    sync = (1 + 2 * 16) * 4
    ws = 3 * slot + 256 + 512 + (sync + 255) // 256 * 256
    Y = gpu_forward(inp, P, act, "fused", ws_bytes=ws)
    ref = oracle.mlp_forward(inp["X"], inp["A"], inp["Wu"], inp["B"], act)
    check(Y, ref, "bf16", "fused ring of 3 slots")


@pytest.mark.parametrize("P", [1, 2, 4, 8])
def test_bf16_independent_of_P(P):
    wl = small("swiglu", "bf16", 512, 512, 8 * 256, P, seed=3)
    inp = make_inputs(wl)
    Y = gpu_forward(inp, P, "swiglu")
    ref = oracle.mlp_forward(inp["X"], inp["A"], inp["Wu"], inp["B"], "swiglu")
    check(Y, ref, "bf16", f"P={P}")


@pytest.mark.parametrize("n,d,f,P,sched", [(4 * 128, 128, 4 * 128, 4, "tsp_ring"),
                                           (8 * 100, 256, 8 * 96, 8, "tsp_ring"),
                                           (8 * 100, 256, 8 * 128, 8, "tsp_ring"),
                                           (2 * 64, 64, 2 * 64, 2, "tsp_ring"),
                                           (4 * 128, 128, 4 * 128, 4, "tsp_ring_fused"),
                                           (8 * 200, 256, 8 * 128, 8, "tsp_ring_fused"),
                                           (2 * 64, 64, 2 * 64, 2, "tsp_ring_fused")])
def test_bf16_tsp_ring_small(n, d, f, P, sched):
    wl = small("swiglu", "bf16", n, d, f, P, seed=11)
    inp = make_inputs(wl)
    Y = gpu_forward(inp, P, "swiglu", sched)
    ref = oracle.mlp_tsp(inp["X"], inp["A"], inp["Wu"], inp["B"], "swiglu", P)
    check(Y, ref, "bf16", "tsp ring")


def test_bf16_row_groups_from_a_small_workspace():
    """A workspace with room for 512 rows of H: the forward runs as two
    one-chunk passes over token rows 0-511 and 512-999 (a ragged last group)."""
    n, d, f, P = 1000, 256, 4 * 256, 4
    wl = small("swiglu", "bf16", n, d, f, P, seed=13)
    inp = make_inputs(wl)
    Y = gpu_forward(inp, P, "swiglu", "weight_shards", ws_bytes=512 * f * 2)
    ref = oracle.mlp_forward(inp["X"], inp["A"], inp["Wu"], inp["B"], "swiglu")
    check(Y, ref, "bf16", "row groups of 512")


def test_bf16_tsp_ring_sequence_shard_groups():
    """A workspace with room for two sequence shards' hidden blocks: the ring
    runs as two launches of two shards, each shard's K loop in its ring order."""
    n, d, f, P = 4 * 128, 128, 4 * 128, 4
    wl = small("swiglu", "bf16", n, d, f, P, seed=12)
    inp = make_inputs(wl)
    ws = 2 * (n // P) * f * 2 + 256
    Y = gpu_forward(inp, P, "swiglu", "tsp_ring", ws_bytes=ws)
    ref = oracle.mlp_tsp(inp["X"], inp["A"], inp["Wu"], inp["B"], "swiglu", P)
    check(Y, ref, "bf16", "tsp ring, 2 shards a launch")


@pytest.mark.parametrize("sched", ["weight_shards", "shard_passes_fused", "fused", "tsp_ring",
                                   "tsp_ring_fused"])
def test_bf16_run_to_run_bitwise_deterministic(sched):
    wl = small("swiglu", "bf16", 1024, 384, 8 * 128, 8, seed=21)
    inp = make_inputs(wl)
    Y1 = gpu_forward(inp, 8, "swiglu", sched)
    Y2 = gpu_forward(inp, 8, "swiglu", sched)
    assert np.array_equal(Y1, Y2)


def test_tsp_mlp_forward_basic_entry_point():
    """tsp_mlp_forward (scratch from cudaMallocAsync) matches the _ex call."""
    wl = small("swiglu", "bf16", 256, 256, 4 * 128, 4, seed=8)
    inp = make_inputs(wl)
    X, A, Wu, B = (to_dev(inp[k]) for k in ("X", "A", "Wu", "B"))
    Y = torch.empty(256, 256, dtype=torch.bfloat16, device="cuda")
    T.tsp_mlp_forward(X, A, Wu, B, 256, 256, 512, 4, "swiglu", Y)
    Y2 = T.mlp_forward(X, A, Wu, B, 4, "swiglu")
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)


# ---------------------------------------------------------------------------- full sizes, sampled


def _full_inputs(wl):
    inp = make_inputs(wl)
    return inp, {k: to_dev(v) for k, v in inp.items()}


def _sampled_check(wl, inp, Y_dev, rows, act="swiglu", sched="weight_shards", P=None):
    P = wl.P if P is None else P
    Y = Y_dev[rows].float().cpu().double().numpy()
    X = inp["X"][rows]
    if sched.startswith("tsp_ring"):
        # the ring result of a row is its sequence shard's ring-ordered sum;
        # within fp64 it equals the unsharded block (pinned in the oracle tests)
        ref = oracle.mlp_forward(X, inp["A"], inp["Wu"], inp["B"], act)
    else:
        ref = oracle.mlp_sharded(X, inp["A"], inp["Wu"], inp["B"], act, P)
    return check(Y, ref, "bf16", f"{wl.name} P={P} {sched}")


@pytest.fixture(scope="module")
def llama8b():
    return _full_inputs(LLAMA8B)


@pytest.mark.parametrize("P,sched", [(8, "weight_shards"), (7, "weight_shards"),
                                     (4, "weight_shards"),
                                     (2, "weight_shards"), (1, "weight_shards"),
                                     (8, "shard_passes_fused"), (8, "fused"), (1, "fused")])
def test_llama8b_shape_sampled_rows(llama8b, P, sched):
    inp, dev = llama8b
    Y = T.mlp_forward(dev["X"], dev["A"], dev["Wu"], dev["B"], P, "swiglu", sched=sched)
    assert T.tsp_poll_device_error() == T.TSP_OK
    # one seeded row in each of the 16 blocks of 256 token rows (every pair row
    # tile of the one row group; every second 128-row tile of the one-CTA fused
    # schedule), plus rows 0 and 4095
    rows = cover_rows(LLAMA8B.n, 256, LLAMA8B.seed)
    _sampled_check(LLAMA8B, inp, Y, rows, sched=sched, P=P)


@pytest.mark.parametrize("sched", ["tsp_ring", "tsp_ring_fused"])
def test_tsp_ring_long_context_sampled_rows(sched):
    inp, dev = _full_inputs(TSP_RING)
    Y = T.mlp_forward(dev["X"], dev["A"], dev["Wu"], dev["B"], TSP_RING.P, "swiglu",
                      sched=sched)
    assert T.tsp_poll_device_error() == T.TSP_OK
    # one seeded row in each of the 128 blocks of 256 token rows (every pair row
    # tile of every sequence shard, so every ring group of sequence shards),
    # plus the first and last row of each of the 8 sequence shards
    ns = TSP_RING.n // TSP_RING.P
    rows = cover_rows(TSP_RING.n, 256, TSP_RING.seed,
                      groups=[(s * ns, (s + 1) * ns) for s in range(TSP_RING.P)])
    assert len(rows) >= 128
    _sampled_check(TSP_RING, inp, Y, rows, sched=sched)


def test_llama70b_shape_sampled_rows():
    inp, dev = _full_inputs(LLAMA70B)
    Y = T.mlp_forward(dev["X"], dev["A"], dev["Wu"], dev["B"], LLAMA70B.P, "swiglu")
    assert T.tsp_poll_device_error() == T.TSP_OK
    # the 70B shape runs as 4 row groups of 2048 tokens (H of a group is 117 MB):
    # one seeded row in each of the 32 blocks of 256 rows (every pair row tile
    # of every group), plus each group's first and last row (0, 2047, 2048,
    # 4095, 4096, 6143, 6144, 8191)
    groups = [(g * 2048, (g + 1) * 2048) for g in range(4)]
    rows = cover_rows(LLAMA70B.n, 256, LLAMA70B.seed, groups=groups)
    assert {4096, 6143} <= set(rows) and len(rows) >= 32
    _sampled_check(LLAMA70B, inp, Y, rows)


@pytest.mark.parametrize("act", ["swiglu", "gelu"])
def test_bf16_down_projection_tail_split(act):
    """80 down-projection tiles of 256 x 256 on 74 CTA pairs: the last wave's
    6 tiles each run as two halves of their K loop on two pairs, the second
    half adding the first's fp32 sum (the tail split).  Compared in full, and
    with the same forward run without the split (a workspace without its
    room), which differs only in the rounding of the split tiles."""
    n, d, f, P = 10 * 256, 8 * 256, 8 * 128, 8
    wl = small(act, "bf16", n, d, f, P, seed=81, w_std=0.03)
    inp = make_inputs(wl)
    Y = gpu_forward(inp, P, act)
    ref = oracle.mlp_forward(inp["X"], inp["A"], inp["Wu"], inp["B"], act)
    check(Y, ref, "bf16", "tail split")
    Y2 = gpu_forward(inp, P, act, ws_bytes=n * f * 2)
    check(Y2, ref, "bf16", "no tail split")
    # tiles run column block by column block: the split ones are the last 6
    # (rows 1024-2559 of columns 1792-2047); every other tile is bit-identical
    assert np.array_equal(Y[:, :1792], Y2[:, :1792])
    assert np.array_equal(Y[:1024], Y2[:1024])
