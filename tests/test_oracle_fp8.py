"""Pins of the oracle's fp8 e4m3 quantisation (oracle/fp8.py), CPU only.

The e4m3 format is fixed by its definition (OCP 8-bit floating point, E4M3):
the value table is checked against values the definition gives directly,
the rounding against torch's float8_e4m3fn conversion (a library routine,
round to nearest even) and against a brute-force nearest-value search.  The
block rule (one scale per 128-row internal block) is checked on its exact
consequences.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8


def test_value_table_follows_the_format():
    v = fp8.e4m3_values()
    assert v[0x00] == 0.0 and np.signbit(v[0x80])
    assert v[0x01] == 2.0 ** -9                   # smallest subnormal
    assert v[0x07] == 7 * 2.0 ** -9               # largest subnormal
    assert v[0x08] == 2.0 ** -6                   # smallest normal
    assert v[0x38] == 1.0                         # exponent field 7 = bias
    assert v[0x3C] == 1.5
    assert v[0x7E] == 448.0 and v[0xFE] == -448.0
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    assert np.isfinite(v).sum() == 254
    fin = v[:0x7F]
    assert (np.diff(fin) > 0).all()               # codes 0..126 increase


def test_rounding_matches_torch_in_range():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.uniform(-448, 448, 100000), rng.standard_normal(50000) * 0.01,
                        rng.standard_normal(50000) * 1e-3]).astype(np.float32)
    got = fp8.e4m3_round(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(got, ref)


def test_midpoints_round_to_even_mantissa():
    v = fp8.e4m3_values()[:0x7F]
    mids = ((v[:-1] + v[1:]) / 2).astype(np.float32)
    codes = fp8.e4m3_round(mids)
    assert (codes & 1 == 0).all()                 # the even neighbour of each tie
    np.testing.assert_array_equal(codes, torch.from_numpy(mids).to(torch.float8_e4m3fn).view(torch.uint8).numpy())


def test_rounding_is_nearest_by_brute_force():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(4000) * 20).astype(np.float32)
    x = x[np.abs(x) <= 448]
    vals = fp8.e4m3_values()
    fin = vals[np.isfinite(vals)]
    best = np.abs(fin[None, :] - x[:, None].astype(np.float64)).min(1)
    got = np.abs(vals[fp8.e4m3_round(x)] - x)
    np.testing.assert_array_equal(got, best)


def test_saturation_above_448():
    x = np.array([448.0, 449.0, 463.9, 464.0, 1e9, -500.0], dtype=np.float32)
    np.testing.assert_array_equal(fp8.e4m3_round(x), [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE])


def test_block_amax_maps_to_448_and_error_is_half_a_step():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((128, 128)) * 3).astype(np.float32)
    codes, scale = fp8.quantize_block(x)
    amax = np.abs(x).max()
    assert scale == np.float32(amax / np.float32(448))
    i = np.unravel_index(np.abs(x).argmax(), x.shape)
    assert codes[i] & 0x7F == 0x7E                # the largest element becomes +-448
    deq = fp8.dequantize(codes, scale)
    # each value lands within half an e4m3 step (relative 2^-4 for normals) of x * inv
    v = np.abs(x.astype(np.float64)) / float(scale)
    step = np.where(v >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(v, 2.0 ** -6))) - 3), 2.0 ** -9)
    assert (np.abs(deq - x) <= 0.5 * step * float(scale) * (1 + 1e-6) + 1e-12).all()


def test_zero_block_has_zero_scale():
    codes, scale = fp8.quantize_block(np.zeros((128, 128), np.float32))
    assert scale == 0 and not codes.any()


def test_scale_invariance_of_codes():
    # multiplying a block by a power of two leaves its codes unchanged and scales its scale
    rng = np.random.default_rng(4)
    x = rng.standard_normal((128, 128)).astype(np.float32)
    c1, s1 = fp8.quantize_block(x)
    c2, s2 = fp8.quantize_block(x * np.float32(8))
    np.testing.assert_array_equal(c1, c2)
    assert s2 == s1 * 8


def test_internal_tiles_cover_the_layout():
    g = oracle.geometry(37 + 8 * 21 * 43, 37, 8, 21, 43)
    tiles = fp8.internal_tiles(g)
    rows = np.concatenate(tiles)
    valid = rows[rows >= 0]
    assert len(tiles) * 128 == len(rows)
    np.testing.assert_array_equal(np.sort(valid), np.arange(g.S))       # every token once
    assert all(len(t) == 128 for t in tiles)
    assert (rows[len(g.prefix):len(g.prefix) + (-len(g.prefix)) % 128] == -1).all()


def test_fp8_oracle_is_close_to_the_native_one():
    # quantisation error of Q, K, V only: small against the output's scale
    from block_sparse_video_rf_b200 import synth
    w = synth.workload("tiny", N=1)
    q, k, v = (t.float().numpy() for t in synth.make_inputs(w))
    ref, mask, _, _ = oracle.rf_sparse_attention(q, k, v, w.layout, w.txt_len, w.latent, w.sparsity)
    got, mask8, _, _ = fp8.rf_sparse_attention_fp8(q, k, v, w.layout, w.txt_len, w.latent, w.sparsity)
    np.testing.assert_array_equal(mask, mask8)
    err = np.abs(got - ref)
    assert err.max() < 0.05 and err.mean() < 5e-3
    assert err.max() > 0          # quantisation does change the result
