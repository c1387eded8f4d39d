"""Planted mistakes in the oracle must fail its pins.

Each case replaces one function of the oracle, for this test only and on
the CPU, with a plausible wrong version (a transposed operand, a tie broken
the other way, a dropped term, a wrong rounding or scale) and runs the pins
that should catch it: at least one must fail.  This shows that the pins fix
the oracle's results rather than merely agreeing with them.
"""

import dataclasses
import json
import math
import os

import numpy as np
import pytest

import oracle
import test_oracle_fp8 as fp8_pins
import test_oracle_pins as pins
from oracle import fp8, rf_v2

ORIG = {n: getattr(rf_v2, n) for n in ("geometry", "block_scores", "topk_mask", "kept_count", "key_set",
                                      "pool_blocks", "_softmax_attend")}
with open(os.path.join(os.path.dirname(__file__), "golden", "geometry_worked_examples.json")) as _f:
    GOLDEN = json.load(_f)


def _raster_transposed_in_tiles(S, txt_len, T, H, W):
    # R1 read as column-major inside each 8x8 tile
    g = ORIG["geometry"](S, txt_len, T, H, W)
    if g.nb == 0:
        return g
    tiles = g.blocks.reshape(g.nb, 2, 8, 8).transpose(0, 1, 3, 2).reshape(g.nb, 128)
    return dataclasses.replace(g, blocks=np.ascontiguousarray(tiles))


def _first_frame_only_whole_blocks(S, txt_len, T, H, W):
    # R3 read as "every token in frame 0" instead of "any token"
    g = ORIG["geometry"](S, txt_len, T, H, W)
    if g.nb == 0:
        return g
    frame = (g.blocks - txt_len) // (H * W)
    return dataclasses.replace(g, first_frame=(frame == 0).all(axis=1))


def _tail_dropped(S, txt_len, T, H, W):
    # R2 read as "the aligned tokens past the last whole block are dropped"
    g = ORIG["geometry"](S, txt_len, T, H, W)
    if len(g.tail) == 0:
        return g
    keep = ~np.isin(g.prefix, g.tail)
    return dataclasses.replace(g, prefix=g.prefix[keep], tail=g.tail[:0])


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
    "raster_transposed_in_tiles": ("geometry", _raster_transposed_in_tiles),
    "first_frame_only_whole_blocks": ("geometry", _first_frame_only_whole_blocks),
    "tail_dropped_not_promoted": ("geometry", _tail_dropped),
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
    (pins.test_worked_geometry_minimax, (GOLDEN,)),
    *[(pins.test_partition_is_a_bijection, args) for args in [(0, 4, 32, 32), (5, 5, 24, 40)]],
    (pins.test_tile_order_by_enumeration, ()),
    (pins.test_odd_tile_count_promotes_last_half_block, ()),
    (pins.test_minimax_first_frame_is_eight, ()),
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


# ---------------------------------------------------------------- e4m3 quantisation (R14)

ORIG8 = {n: getattr(fp8, n) for n in ("e4m3_round", "quantize_block")}
_POS = fp8.e4m3_values()[:0x7F]          # codes 0x00 .. 0x7E: the finite non-negative values, ascending


def _codes_from_magnitude_index(idx, x):
    x = np.asarray(x, dtype=np.float64)
    return (np.asarray(idx, dtype=np.int64) | np.where(np.signbit(x), 0x80, 0)).astype(np.uint8)


def _toward_zero(x):
    a = np.minimum(np.abs(np.asarray(x, dtype=np.float64)), _POS[-1])
    return _codes_from_magnitude_index(np.searchsorted(_POS, a, side="right") - 1, x)


def _ties_away_from_zero(x):
    a = np.minimum(np.abs(np.asarray(x, dtype=np.float64)), _POS[-1])
    lo = np.searchsorted(_POS, a, side="right") - 1
    hi = np.minimum(lo + 1, len(_POS) - 1)
    up = (_POS[hi] - a) <= (a - _POS[lo])
    return _codes_from_magnitude_index(np.where(up, hi, lo), x)


def _no_saturation(x):
    codes = ORIG8["e4m3_round"](x)
    over = np.abs(np.asarray(x, dtype=np.float64)) > fp8.E4M3_MAX
    return np.where(over, codes | 0x7F, codes).astype(np.uint8)


def _scale_of_127(x):
    xf = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(xf))) if xf.size else np.float32(0.0)
    if amax == 0:
        return np.zeros(xf.shape, dtype=np.uint8), np.float32(0.0)
    return fp8.e4m3_round((xf * np.float32(np.float32(127.0) / amax)).astype(np.float32)), np.float32(amax / 127.0)


MISTAKES8 = {
    "rounding_toward_zero": ("e4m3_round", _toward_zero),
    "ties_away_from_zero": ("e4m3_round", _ties_away_from_zero),
    "no_saturation_above_448": ("e4m3_round", _no_saturation),
    "scale_of_127": ("quantize_block", _scale_of_127),
}
PINS8 = [
    (fp8_pins.test_rounding_matches_torch_in_range, ()),
    (fp8_pins.test_midpoints_round_to_even_mantissa, ()),
    (fp8_pins.test_rounding_is_nearest_by_brute_force, ()),
    (fp8_pins.test_saturation_above_448, ()),
    (fp8_pins.test_block_amax_maps_to_448_and_error_is_half_a_step, ()),
    (fp8_pins.test_zero_block_has_zero_scale, ()),
    (fp8_pins.test_scale_invariance_of_codes, ()),
]


def _failures8():
    names = []
    for pin, args in PINS8:
        try:
            pin(*args)
        except Exception:
            names.append(pin.__name__)
    return names


def test_the_fp8_pins_pass_on_the_oracle_as_it_stands():
    assert _failures8() == []


@pytest.mark.parametrize("mistake", sorted(MISTAKES8))
def test_a_planted_fp8_mistake_fails_a_pin(mistake, monkeypatch):
    name, wrong = MISTAKES8[mistake]
    monkeypatch.setattr(fp8, name, wrong)
    assert _failures8(), f"no pin caught {mistake}"
