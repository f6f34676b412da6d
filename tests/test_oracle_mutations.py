"""The oracle's pins catch plausible mistakes.

Each case plants one plausible mistake in a temporary copy of the oracle's C
source (a wrong sign, a dropped term, a wrong index or range, a lost
accumulation), compiles it on the CPU, and checks that at least one pin of the
battery below fails.  The battery uses the same independent references as
``test_oracle_pins.py``: the hand-worked 2x2 closed forms, P / order / ring
invariance, and the finite-difference check of the backward.
"""
import json
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "oracle", "tspmlp_oracle.c")

MUTATIONS = {
    "sigmoid_sign": ("return 1.0 / (1.0 + exp(-g));", "return 1.0 / (1.0 + exp(g));"),
    "gelu_scale": ("erf(z / sqrt(2.0))", "erf(z / 2.0)"),
    "silu_grad_dropped_term": ("s * (1.0 + gj * (1.0 - s))", "s * (1.0 - s)"),
    "gelu_grad_dropped_term": ("(std_normal_cdf(gj) + gj * std_normal_pdf(gj))",
                               "std_normal_cdf(gj)"),
    "down_proj_row_index": ("const double* brow = B + j * d;\n        for (int64_t c = 0; c < d; ++c) y[c] += hj * brow[c];",
                            "const double* brow = B + (j - j0) * d;\n        for (int64_t c = 0; c < d; ++c) y[c] += hj * brow[c];"),
    "shard_range_short": ("row_block(X + i * d, A, Wu, B, act, d, f, (int64_t)w * fs,\n                              (int64_t)(w + 1) * fs, g, u, h, y);\n                    for (int64_t c = 0; c < d; ++c) yi[c] += y[c];\n                }\n            }\n        }\n        free(g);\n        free(u);\n        free(h);\n        free(y);\n    }\n    return err;\n}\n\n/* Folded",
                          "row_block(X + i * d, A, Wu, B, act, d, f, (int64_t)w * fs,\n                              (int64_t)(w + 1) * fs - 1, g, u, h, y);\n                    for (int64_t c = 0; c < d; ++c) yi[c] += y[c];\n                }\n            }\n        }\n        free(g);\n        free(u);\n        free(h);\n        free(y);\n    }\n    return err;\n}\n\n/* Folded"),
    "sharded_overwrite": ("for (int64_t c = 0; c < d; ++c) yi[c] += y[c];\n                }\n            }\n        }\n        free(g);\n        free(u);\n        free(h);\n        free(y);\n    }\n    return err;\n}\n\n/* Folded",
                          "for (int64_t c = 0; c < d; ++c) yi[c] = y[c];\n                }\n            }\n        }\n        free(g);\n        free(u);\n        free(h);\n        free(y);\n    }\n    return err;\n}\n\n/* Folded"),
    "ring_stuck_on_one_shard": ("(s - t) % P + P) % P : (s + t) % P;", "(s - t) % P + P) % P : (s) % P;"),
    "dX_drops_up_branch": ("for (int64_t j = 0; j < f; ++j) s += dU[i * f + j] * urow[j];",
                           "for (int64_t j = 0; j < f; ++j) s += 0.0 * dU[i * f + j] * urow[j];"),
    "dWd_uses_preactivation": ("H[i * f + j] = gj * s * u[j];", "H[i * f + j] = gj * u[j];"),
    # reads the pre-activation weight as if it were stored transposed
    "preact_transposed_weight": ("for (int64_t j = 0; j < w; ++j) g[j] += xk * arow[j];",
                                 "for (int64_t j = 0; j < w; ++j) g[j] += xk * A[((j0 + j) * d + k) % (d * f)];"),
}


def _battery(lib_path):
    """Run the pins against the library at lib_path; return the names of the
    pins that fail."""
    saved = oracle._lib
    oracle._lib = oracle.bind(lib_path)
    failed = []
    try:
        import test_oracle_pins as T
        with open(T.GOLDEN) as fh:
            g2 = json.load(fh)
        checks = [
            ("gelu_2x2", lambda: T.test_gelu_2x2_forward(g2)),
            ("gelu_2x2_partials", lambda: T.test_gelu_2x2_shard_partials(g2)),
            ("swiglu_2x2", lambda: T.test_swiglu_2x2_forward(g2)),
            ("swiglu_2x2_bwd", lambda: T.test_swiglu_2x2_backward(g2)),
            ("gelu_2x2_bwd", lambda: T.test_gelu_2x2_backward(g2)),
            ("P_invariance_gelu", lambda: T.test_independent_of_P("gelu")),
            ("P_invariance_swiglu", lambda: T.test_independent_of_P("swiglu")),
            ("tsp_gelu", lambda: T.test_tsp_ring_equals_unsharded_and_either_direction("gelu")),
            ("fd_swiglu", lambda: T.test_backward_central_differences("swiglu")),
            ("fd_gelu", lambda: T.test_backward_central_differences("gelu")),
        ]
        for name, fn in checks:
            try:
                fn()
            except Exception:  # an AssertionError or a rejected call
                failed.append(name)
    finally:
        oracle._lib = saved
    return failed


@pytest.fixture(scope="module")
def source():
    with open(SRC) as fh:
        return fh.read()


def test_unmutated_oracle_passes_the_battery(tmp_path):
    lib = tmp_path / "liboracle_clean.so"
    shutil.copy(oracle.build(), lib)
    assert _battery(str(lib)) == []


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, source, tmp_path):
    old, new = MUTATIONS[name]
    assert source.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = source.replace(old, new, 1)
    src = tmp_path / "mut.c"
    lib = tmp_path / f"libmut_{name}.so"
    src.write_text(mutated)
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC", "-o",
                    str(lib), str(src), "-lm"], check=True)
    failed = _battery(str(lib))
    assert failed, f"planted mistake {name!r} passed every pin"
