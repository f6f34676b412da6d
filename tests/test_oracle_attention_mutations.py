"""The attention oracle's pins catch plausible mistakes.

Each case plants one plausible mistake in a temporary copy of
oracle/attention.py (a wrong scale or mask, a dropped rescale in the running
softmax merge, a stuck ring, a wrong head slice, a lost accumulation, a wrong
operand) and checks that at least one pin of test_oracle_attention_pins.py
fails against it."""
import importlib.util
import json
import os

import pytest

import test_oracle_attention_pins as T

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "oracle", "attention.py")

MUTATIONS = {
    "scale_by_dh": ("s = (q @ k.T) / math.sqrt(dh)", "s = (q @ k.T) / dh"),
    "causal_mask_off_by_one": ("k_pos[None, :] > q_pos[:, None]", "k_pos[None, :] >= q_pos[:, None]"),
    "merge_drops_acc_rescale": ("acc = acc * scale_old + e @ V[ku, c]", "acc = acc + e @ V[ku, c]"),
    "merge_drops_sum_rescale": ("l = l * scale_old + e.sum", "l = l + e.sum"),
    "ring_stuck_on_own_shard": ("return (s + t) % P", "return s % P"),
    "head_slice_wrong": ("c = slice(h * dh, (h + 1) * dh)\n        s = _scores",
                         "c = slice(h, h + dh)\n        s = _scores"),
    "partial_outputs_overwrite": ("Y[r] += Osw @ Wo[cols, :]", "Y[r] = Osw @ Wo[cols, :]"),
    "output_rows_of_first_shard": ("Y[r] += Osw @ Wo[cols, :]", "Y[r] += Osw @ Wo[:cw, :]"),
    "keys_as_values": ("O[:, c] = (e @ V[:, c])", "O[:, c] = (e @ K[:, c])"),
    "max_subtracted_wrong_way": ("e = np.exp(s - m)", "e = np.exp(m - s)"),
    "keys_projected_with_wq": ("Kw[r] = X[r] @ Wk[:, cols]", "Kw[r] = X[r] @ Wq[:, cols]"),
    "visited_shard_positions": ("np.arange(u * ns, (u + 1) * ns), dh, causal)",
                                "np.arange(s * ns, (s + 1) * ns), dh, causal)"),
}


def _battery(module):
    saved = T.A
    T.A = module
    failed = []
    try:
        with open(T.GOLDEN) as fh:
            g2 = json.load(fh)
        checks = [
            ("two_token", lambda: [T.test_two_token_block(g2, c) for c in (False, True)]),
            ("two_token_tsp", lambda: [T.test_two_token_tsp_schedule(g2, c) for c in (False, True)]),
            ("sdpa", lambda: [T.test_core_equals_torch_sdpa_fp64(33, 16, 4, c) for c in (False, True)]),
            ("brute", lambda: [T.test_brute_force_tiny(6, 6, 3, 3, c) for c in (False, True)]),
            ("P_invariance", lambda: [T.test_tsp_independent_of_P_and_equal_to_plain(c)
                                      for c in (False, True)]),
            ("order_invariance", lambda: [T.test_tsp_independent_of_visiting_and_shard_order(c)
                                          for c in (False, True)]),
            ("ring", T.test_ring_visits_every_shard_once_starting_at_its_own),
            ("causal_first_row", T.test_causal_first_row_is_its_own_value),
            ("uniform", T.test_zero_queries_attend_uniformly),
            ("one_hot", T.test_dominant_score_selects_one_value),
        ]
        for name, fn in checks:
            try:
                fn()
            except Exception:  # an AssertionError or a rejected call
                failed.append(name)
    finally:
        T.A = saved
    return failed


def _load(path, name):
    spec = importlib.util.spec_from_file_location(name, path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.fixture(scope="module")
def source():
    with open(SRC) as fh:
        return fh.read()


def test_unmutated_oracle_passes_the_battery():
    assert _battery(_load(SRC, "attention_clean")) == []


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, source, tmp_path):
    old, new = MUTATIONS[name]
    assert source.count(old) >= 1, f"mutation anchor for {name} not found"
    path = tmp_path / f"attention_{name}.py"
    path.write_text(source.replace(old, new, 1))
    failed = _battery(_load(str(path), f"attention_{name}"))
    assert failed, f"planted mistake {name!r} passed every pin"
