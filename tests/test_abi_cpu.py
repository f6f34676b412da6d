"""The C-ABI library builds, loads and exports every symbol include/tspmlp.h
declares; host-side logic (workspace sizing, argument validation, status
strings) behaves as the header documents.  No GPU is needed: every call here
returns before touching a device."""
import ctypes
import os
import re

import pytest

import sequence_transformer_mlp_b200 as T

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tspmlp.h")


def declared_symbols():
    with open(HEADER) as fh:
        text = fh.read()
    return re.findall(r"TSP_API\s+[\w\s\*]+?\b(tsp_\w+)\s*\(", text)


@pytest.fixture(scope="module")
def lib():
    from sequence_transformer_mlp_b200 import build
    build.build()
    return T.load()


def test_header_declares_the_api():
    syms = set(declared_symbols())
    assert {"tsp_mlp_forward", "tsp_mlp_forward_ex", "tsp_mlp_backward", "tsp_mlp_backward_ex",
            "tsp_mlp_workspace_size", "tsp_status_string", "tsp_poll_device_error",
            "tsp_mlp_saved_size", "tsp_mlp_forward_train", "tsp_mlp_backward_saved",
            "tsp_mlp_backward_saved_workspace_size"} <= syms


def test_header_is_plain_c(tmp_path):
    """The boundary is a C ABI: the header compiles as strict C99 on its own
    (no C++ or CUDA types in the declarations) and as C++."""
    import shutil
    import subprocess
    src = tmp_path / "use_header.c"
    src.write_text('#include "tspmlp.h"\nint main(void) { return (int)TSP_OK; }\n')
    inc = os.path.join(ROOT, "include")
    for cc, std in (("gcc", "-std=c99"), ("g++", "-std=c++17")):
        if shutil.which(cc) is None:
            pytest.skip(f"{cc} not found")
        flags = [std, "-Wall", "-Wextra", "-Werror", "-pedantic"]
        if cc == "g++":
            flags += ["-x", "c++"]
        subprocess.run([cc, *flags, "-I", inc, "-c", str(src), "-o", str(tmp_path / "use.o")],
                       check=True)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings(lib):
    for code, name in T.STATUS_NAMES.items():
        s = T.tsp_status_string(code)
        assert isinstance(s, str) and s
    assert T.tsp_status_string(0) == "ok"
    assert T.tsp_status_string(99) == "unknown status"


def _a256(b):
    return (b + 255) // 256 * 256


# the one-chunk passes' room for the down projection's tail split: the fp32
# partial sums of up to 64 split 256 x 256 tiles and one flag per epilogue warp
SPLIT = 64 * 256 * 256 * 4 + 256 + 64 * 8 * 4 + 256


def test_workspace_sizes_follow_the_schedule(lib):
    # fp32 weight-shard schedule: the hidden block of every shard in one chunk
    # (Y accumulates in place only when there are several chunks)
    assert T.tsp_mlp_workspace_size(64, 128, 512, 2, "gelu", "f32") == 64 * 512 * 4
    # fp32 TSP ring: one ring step's hidden block for all sequence shards
    assert T.tsp_mlp_workspace_size(64, 128, 512, 2, "gelu", "f32", "tsp_ring") == 64 * 256 * 4
    # bf16 fused schedule: an H ring of row-block slots (128 x d_ff) and the
    # per-row-block counters; 2 row blocks -> 2 slots
    assert T.tsp_mlp_workspace_size(256, 64, 512, 1, "swiglu", "bf16", "fused") == \
        _a256(2 * 128 * 512 * 2) + _a256((1 + 2 * 2) * 4)
    # Llama-3-8B shape: 32 row blocks in groups of 8, ring of 3 groups (24 slots)
    n, d, f, P = 4096, 4096, 14336, 8
    assert T.tsp_mlp_workspace_size(n, d, f, P, "swiglu", "bf16", "fused") == \
        _a256(24 * 128 * f * 2) + _a256((1 + 2 * 32) * 4)
    # pass schedule (the default): chunks of whole shards within the 512 MB
    # hidden budget -- here all eight shards in one chunk, so no fp32
    # accumulator; the one-launch form holds two H chunk buffers within 128 MB
    # (2 chunks of 4 shards), the accumulator and the dependency counters
    # (2 chunks x 16 row pairs)
    ws = T.tsp_mlp_workspace_size(n, d, f, P, "swiglu", "bf16", "shard_passes")
    acc = n * d * 4
    assert ws == T.tsp_mlp_workspace_size(n, d, f, P, "swiglu", "bf16") == n * f * 2 + SPLIT
    assert T.tsp_mlp_workspace_size(n, d, f, P, "swiglu", "bf16", "shard_passes_fused") == \
        2 * (n * f // 2 * 2) + acc + _a256((1 + 2 * 2 * 16) * 4)
    # H larger than the 128 MB row-group budget: equal groups of token rows
    # (multiples of 256), each a one-chunk pass -- 70B shape: 4 groups of 2048
    # rows; 32768 tokens of the 8B shape: 8 groups of 4096 rows
    assert T.tsp_mlp_workspace_size(8192, 8192, 28672, 8, "swiglu", "bf16") == \
        2048 * 28672 * 2 + SPLIT
    assert T.tsp_mlp_workspace_size(32768, d, f, P, "swiglu", "bf16") == 4096 * f * 2 + SPLIT
    # single chunk: no accumulator
    assert T.tsp_mlp_workspace_size(256, 64, 512, 1, "swiglu", "bf16", "shard_passes") == \
        256 * 512 * 2 + SPLIT
    # TSP ring fused: 256 row blocks (8 sequence shards of 32), ring of 24 slots;
    # TSP ring passes: sequence shards per launch within the hidden budget + accumulator
    wsr = T.tsp_mlp_workspace_size(32768, d, f, P, "swiglu", "bf16", "tsp_ring_fused")
    assert wsr == _a256(24 * 128 * f * 2) + _a256((1 + 2 * 256) * 4)
    # TSP ring passes with 64-multiple shards: whole-d_ff hidden blocks of as
    # many sequence shards as fit 512 MB (4 of 117 MB), no accumulator
    assert T.tsp_mlp_workspace_size(32768, d, f, P, "swiglu", "bf16", "tsp_ring") == \
        4 * 4096 * f * 2
    # ... otherwise one ring step's shard blocks within the budget + the accumulator
    wsr2 = T.tsp_mlp_workspace_size(8 * 100, 256, 8 * 96, 8, "swiglu", "bf16", "tsp_ring")
    assert wsr2 == _a256(8 * 100 * 96 * 2) + _a256(800 * 256 * 4)
    # fused schedules need bf16; the fused ring needs 64-multiple shards
    out = ctypes.c_size_t(0)
    assert lib.tsp_mlp_workspace_size(64, 64, 128, 1, 1, 1, 3, 0, ctypes.byref(out)) == 2
    assert lib.tsp_mlp_workspace_size(8 * 100, 256, 8 * 96, 8, 1, 0, 4, 0, ctypes.byref(out)) == 2
    # backward: H, dG, dU chunk buffers and the fp32 dX accumulator
    # backward: bf16 H, dG, dU and fp32 dH for all hidden units (one chunk
    # within the 1 GiB budget, so no fp32 dX accumulator)
    wsb = T.tsp_mlp_workspace_size(n, d, f, P, "swiglu", "bf16", backward=True)
    assert wsb == 3 * n * f * 2 + n * f * 4


@pytest.mark.parametrize("args,code", [
    ((0, 64, 128, 1, "gelu", "bf16"), 1),          # n <= 0
    ((64, 64, 130, 4, "gelu", "bf16"), 2),         # d_ff % P
    ((64, 60, 128, 1, "gelu", "bf16"), 2),         # d_model % 8 for bf16
    ((64, 64, 128 * 3, 3, "gelu", "bf16"), 0),     # fine: d_ff/P = 128
    ((64, 64, 108, 3, "gelu", "bf16"), 2),         # (d_ff/P) % 8 for bf16 (36)
    ((64, 60, 120, 3, "gelu", "f32"), 0),          # fp32 takes any sizes
    ((64, 64, 128, 5000, "gelu", "f32"), 2),       # P too large
])
def test_workspace_size_validation(lib, args, code):
    out = ctypes.c_size_t(0)
    n, d, f, P, act, dt = args
    s = lib.tsp_mlp_workspace_size(n, d, f, P, T.ACT[act], T.DTYPE[dt], 0, 0, ctypes.byref(out))
    assert s == code


def test_tsp_ring_needs_divisible_tokens(lib):
    out = ctypes.c_size_t(0)
    assert lib.tsp_mlp_workspace_size(100, 64, 128, 8, 1, 0, 1, 0, ctypes.byref(out)) == 2
    assert lib.tsp_mlp_workspace_size(96, 64, 128, 8, 1, 0, 1, 0, ctypes.byref(out)) == 0


def test_bad_pointers_are_rejected_before_any_device_call(lib):
    A, B, X, Y, U = 0x100000, 0x200000, 0x300000, 0x400000, 0x500000
    # gelu with an up weight, swiglu without one, missing output
    assert T.tsp_mlp_forward(X, A, U, B, 64, 64, 128, 1, "gelu", Y, stream=0, check=False) == 1
    assert T.tsp_mlp_forward(X, A, None, B, 64, 64, 128, 1, "swiglu", Y, stream=0,
                             check=False) == 1
    assert T.tsp_mlp_forward(X, A, None, B, 64, 64, 128, 1, "gelu", None, stream=0,
                             check=False) == 1
    # Y overlapping X
    assert T.tsp_mlp_forward_ex(X, A, None, B, 64, 64, 128, 1, "gelu", "bf16", "weight_shards",
                                X + 64, 0x900000, 1 << 20, stream=0, check=False) == 1
    # misaligned bf16 operand
    assert T.tsp_mlp_forward_ex(X + 2, A, None, B, 64, 64, 128, 1, "gelu", "bf16",
                                "weight_shards", Y, 0x900000, 1 << 20, stream=0,
                                check=False) == 2
    # workspace too small / missing
    assert T.tsp_mlp_forward_ex(X, A, None, B, 64, 64, 128, 1, "gelu", "bf16", "weight_shards", Y,
                                0x900000, 16, stream=0, check=False) == 6
    assert T.tsp_mlp_forward_ex(X, A, None, B, 64, 64, 128, 1, "gelu", "bf16", "weight_shards", Y,
                                None, 0, stream=0, check=False) == 6
    # backward: dW_up must be NULL for gelu and given for swiglu; outputs must not alias
    dX, g1, g2, g3 = 0x600000, 0x700000, 0x800000, 0xA00000
    assert T.tsp_mlp_backward(X, A, None, B, Y, 64, 64, 128, 1, "gelu", dX, g1, g2, g3, stream=0,
                              check=False) == 1
    assert T.tsp_mlp_backward(X, A, U, B, Y, 64, 64, 128, 1, "swiglu", dX, g1, None, g3,
                              stream=0, check=False) == 1
    assert T.tsp_mlp_backward_ex(X, A, U, B, Y, 64, 64, 128, 1, "swiglu", dX, g1, g1, g3,
                                 0xB00000, 1 << 30, stream=0, check=False) == 1


def test_training_pair_sizes(lib):
    # saved activations: bf16 H, then bf16 S1 (and S2 for SwiGLU) over whole
    # 32-row blocks, each region 256-byte aligned
    n, d, f, P = 4096, 4096, 14336, 8
    # (and the down projection's tail-split scratch, as the forward's workspace)
    assert T.tsp_mlp_saved_size(n, d, f, P, "swiglu") == n * f * 2 + 2 * n * f * 2 + SPLIT
    assert T.tsp_mlp_saved_size(n, d, f, P, "gelu") == n * f * 2 + n * f * 2 + SPLIT
    # (the factor regions hold whole 32-row blocks)
    assert T.tsp_mlp_saved_size(3, 16, 8 * 3, 3, "swiglu") == \
        _a256(3 * 24 * 2) + 2 * _a256(32 * 24 * 2) + SPLIT
    # the backward from saved activations needs only dG (dU) chunk buffers:
    # one chunk of all hidden units within the 1 GiB budget
    assert T.tsp_mlp_backward_saved_workspace_size(n, d, f, P, "swiglu") == 2 * n * f * 2
    assert T.tsp_mlp_backward_saved_workspace_size(n, d, f, P, "gelu") == n * f * 2
    # 32768 tokens: 2 x 32768 x 14336 x 2 B is above 1 GiB, so chunks of whole
    # shards (4 of the 8) plus the fp32 dX accumulator
    n2 = 32768
    ws = T.tsp_mlp_backward_saved_workspace_size(n2, d, f, P, "swiglu")
    per_col = n2 * 2 * 2
    cols = (1 << 30) // per_col // 128 * 128
    G = max(g for g in (1, 2, 4, 8) if g * (f // P) <= cols)
    assert ws == 2 * n2 * G * (f // P) * 2 + n2 * d * 4


def test_training_pair_rejects_bad_buffers(lib):
    A, B, X, Y, U = 0x100000, 0x200000, 0x300000, 0x400000, 0x500000
    n, d, f, P = 64, 64, 128, 1
    need = T.tsp_mlp_saved_size(n, d, f, P, "swiglu")
    S = 0x1000000
    fw = T.tsp_mlp_forward_train
    assert fw(X, A, U, B, n, d, f, P, "swiglu", Y, None, need, stream=0, check=False) == 1
    assert fw(X, A, U, B, n, d, f, P, "swiglu", Y, S, need - 1, stream=0, check=False) == 1
    assert fw(X, A, U, B, n, d, f, P, "swiglu", Y, S + 16, need, stream=0, check=False) == 1
    assert fw(X, A, U, B, n, d, f, P, "swiglu", Y, X, need, stream=0, check=False) == 1
    assert fw(X, A, None, B, n, d, f, P, "swiglu", Y, S, need, stream=0, check=False) == 1
    dX, g1, g2, g3, W = 0x600000, 0x700000, 0x800000, 0xA00000, 0x2000000
    ws = T.tsp_mlp_backward_saved_workspace_size(n, d, f, P, "swiglu")
    bw = T.tsp_mlp_backward_saved
    assert bw(X, A, U, B, Y, None, need, n, d, f, P, "swiglu", dX, g1, g2, g3, W, ws, stream=0,
              check=False) == 1
    assert bw(X, A, U, B, Y, S, need - 1, n, d, f, P, "swiglu", dX, g1, g2, g3, W, ws, stream=0,
              check=False) == 1
    assert bw(X, A, U, B, Y, S, need, n, d, f, P, "swiglu", dX, g1, g2, g3, None, 0, stream=0,
              check=False) == 6
    assert bw(X, A, U, B, Y, S, need, n, d, f, P, "swiglu", dX, g1, g2, g3, W, 16, stream=0,
              check=False) == 6
    # an output or the workspace inside the saved buffer
    assert bw(X, A, U, B, Y, S, need, n, d, f, P, "swiglu", S + 256, g1, g2, g3, W, ws, stream=0,
              check=False) == 1
    assert bw(X, A, U, B, Y, S, need, n, d, f, P, "swiglu", dX, g1, g2, g3, S, ws, stream=0,
              check=False) == 1


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(ImportError):
        T.load(str(tmp_path / "nope.so"))


def test_attention_workspace_and_shape_rules(lib):
    # Q, K, V, O: [n][d] bf16 each, 256-byte aligned
    assert T.tsp_attn_workspace_size(32768, 4096, 32, 8) == 4 * 32768 * 4096 * 2
    assert T.tsp_attn_workspace_size(3, 128, 1, 1) == 4 * _a256(3 * 128 * 2)
    out = ctypes.c_size_t(0)
    # head dimension 128 only; tokens a multiple of P; heads a multiple of P
    assert lib.tsp_attn_workspace_size(64, 4096, 64, 8, ctypes.byref(out)) == 2
    assert lib.tsp_attn_workspace_size(100, 1024, 8, 8, ctypes.byref(out)) == 2
    assert lib.tsp_attn_workspace_size(96, 1024, 8, 3, ctypes.byref(out)) == 2
    assert lib.tsp_attn_workspace_size(0, 1024, 8, 8, ctypes.byref(out)) == 1
    assert lib.tsp_attn_workspace_size(64, 1024, 8, 8, None) == 1


def test_attention_bad_arguments_are_rejected_before_any_device_call(lib):
    X, Wq, Wk, Wv, Wo, Y, W = (k << 32 for k in range(1, 8))
    n, d, h, P = 256, 256, 2, 2
    ws = T.tsp_attn_workspace_size(n, d, h, P)
    fw = T.tsp_attn_forward
    assert fw(None, Wq, Wk, Wv, Wo, n, d, h, P, True, Y, W, ws, stream=0, check=False) == 1
    assert fw(X, Wq, Wk, Wv, Wo, n, d, h, P, True, X + 64, W, ws, stream=0, check=False) == 1
    assert fw(X + 2, Wq, Wk, Wv, Wo, n, d, h, P, True, Y, W, ws, stream=0, check=False) == 2
    assert fw(X, Wq, Wk, Wv, Wo, n, d, h, P, True, Y, W, ws - 1, stream=0, check=False) == 6
    assert fw(X, Wq, Wk, Wv, Wo, n, d, h, P, True, Y, W + 16, ws, stream=0, check=False) == 6
    assert fw(X, Wq, Wk, Wv, Wo, n, d, h, P, True, Y, X, ws, stream=0, check=False) == 1
    assert fw(X, Wq, Wk, Wv, Wo, n, d, h, 4, True, Y, W, ws, stream=0, check=False) == 2
    core = T.tsp_attn_core
    assert core(X, Wq, Wk, n, d, h, P, False, None, stream=0, check=False) == 1
    assert core(X, Wq, Wk, n, d, h, P, False, Wq + 512, stream=0, check=False) == 1
    assert core(X, Wq, Wk, n, 192, h, P, False, Y, stream=0, check=False) == 2
    assert core(X, Wq, Wk, 255, d, h, P, False, Y, stream=0, check=False) == 2
