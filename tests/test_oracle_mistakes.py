"""Planted mistakes in the oracle must fail its pins.

Each case replaces one function of the oracle, for this test only and on
the CPU, with a plausible wrong version (a transposed operand, a tie broken
the other way, a dropped term, a wrong rounding or scale) and runs the pins
that should catch it: at least one must fail.  This shows that the pins fix
the oracle's results rather than merely agreeing with them.
"""

import math

import numpy as np
import pytest

import oracle
import test_oracle_pins as pins
from oracle import rf_v2

ORIG = {n: getattr(rf_v2, n) for n in ("block_scores", "topk_mask", "kept_count", "key_set", "pool_blocks",
                                      "_softmax_attend")}


def _ties_to_the_higher_index(scores, k, first_frame, first_frame_cols=None):
    cols = first_frame if first_frame_cols is None else first_frame_cols
    mask, margin = ORIG["topk_mask"](np.ascontiguousarray(scores[:, ::-1]), k, first_frame,
                                     np.ascontiguousarray(cols[::-1]))
    return np.ascontiguousarray(mask[:, ::-1]), margin


def _prefix_keys_left_out(g, mask_bn, row_block, gk=None):
    keys = ORIG["key_set"](g, mask_bn, row_block, gk)
    if row_block is None:
        return keys
    return np.setdiff1d(keys, (gk if gk is not None else g).prefix)


MISTAKES = {
    "scores_transposed": ("block_scores", lambda qbar, kbar: ORIG["block_scores"](kbar, qbar)),
    "ties_to_the_higher_index": ("topk_mask", _ties_to_the_higher_index),
    "first_frame_columns_not_forced": (
        "topk_mask", lambda scores, k, ff, ffc=None: ORIG["topk_mask"](scores, k, ff, np.zeros(scores.shape[1], bool))),
    "first_frame_rows_not_dense": (
        "topk_mask", lambda scores, k, ff, ffc=None: ORIG["topk_mask"](scores, k, np.zeros_like(ff),
                                                                      ff if ffc is None else ffc)),
    "dropped_count_rounded_up": ("kept_count", lambda nb, s: nb - min(nb, math.ceil(s * nb - 1e-6))),
    "prefix_keys_left_out": ("key_set", _prefix_keys_left_out),
    "block_sums_not_means": ("pool_blocks", lambda x, blocks: ORIG["pool_blocks"](x, blocks) * blocks.shape[1]),
    "softmax_scale_squared": ("_softmax_attend", lambda q, k, v, scale: ORIG["_softmax_attend"](q, k, v, scale * scale)),
}

# the pins run against each mistake (pins with parameters: a few of their cases)
PINS = [
    (pins.test_kept_count_fixed_points, ()),
    (pins.test_block_means_of_constant_and_index_rows, ()),
    *[(pins.test_topk_matches_exhaustive_search, (seed,)) for seed in range(4)],
    (pins.test_topk_first_frame_rows_and_columns, ()),
    (pins.test_sparsity_zero_equals_dense_sdpa, ()),
    (pins.test_one_hot_value_probe_reads_exactly_the_expected_blocks, ()),
    (pins.test_constant_value_gives_constant_output, ()),
]


def _failures():
    names = []
    for pin, args in PINS:
        try:
            pin(*args)
        except Exception:   # an assertion, or the wrong version breaking the pin's own code
            names.append(pin.__name__)
    return names


def test_the_pins_pass_on_the_oracle_as_it_stands():
    assert _failures() == []


@pytest.mark.parametrize("mistake", sorted(MISTAKES))
def test_a_planted_mistake_fails_a_pin(mistake, monkeypatch):
    name, wrong = MISTAKES[mistake]
    monkeypatch.setattr(rf_v2, name, wrong)
    if hasattr(oracle, name):
        monkeypatch.setattr(oracle, name, wrong)
    failed = _failures()
    assert failed, f"no pin caught {mistake}"
