"""Failure detection on the GPU without a fault: every wait in the library's
kernels is bounded.  The self-test makes a wait run out (an mbarrier nothing
arrives on; a pipeline stage whose loads were left out), the kernel returns,
the host reads TSP_ERR_TIMEOUT from the device error word, and the context
stays usable for a normal forward pass afterwards."""
import time

import numpy as np
import pytest

import oracle
import sequence_transformer_mlp_b200 as T
from workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu


def _forward_still_correct():
    wl = Workload("after_timeout", "swiglu", "bf16", 256, 128, 2 * 128, 2, seed=17, w_std=0.05)
    inp = make_inputs(wl)
    dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    Y = T.mlp_forward(dev["X"], dev["A"], dev["Wu"], dev["B"], 2, "swiglu")
    assert T.tsp_poll_device_error() == T.TSP_OK
    ref = oracle.mlp_forward(inp["X"], inp["A"], inp["Wu"], inp["B"], "swiglu")
    g = Y.float().cpu().double().numpy()
    assert np.linalg.norm(g - ref) / np.linalg.norm(ref) <= 5e-3


@pytest.mark.parametrize("mode", [0, 1])
def test_bounded_wait_reports_timeout_and_context_survives(mode):
    T.load()
    assert T.tsp_poll_device_error() == T.TSP_OK
    t0 = time.time()
    T.tsp_selftest_timeout(mode)
    assert T.tsp_poll_device_error() == T.TSP_ERR_TIMEOUT
    elapsed = time.time() - t0
    assert 1.5 < elapsed < 30.0, elapsed
    assert T.tsp_poll_device_error() == T.TSP_OK  # the word was cleared
    _forward_still_correct()


def test_selftest_rejects_unknown_mode():
    T.load()
    assert T.load().tsp_selftest_timeout(7, None) == 1
