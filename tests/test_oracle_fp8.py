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


# ---------------------------------------------------------------- the e4m3 rounding of P (R15)

def _e4m3(x: np.ndarray) -> np.ndarray:
    """fp32 -> nearest e4m3 value by torch's float8_e4m3fn conversion (a library routine, RNE)."""
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).double().numpy()


def _bf16(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def _row_case(seed: int, spread: float, ref_drop: float, n_tiles: int = 8, D: int = 16, R: int = 64):
    """Random rows of scores (log2 units) over n_tiles x 128 keys, V quantised
    per 128-key tile with torch's e4m3 conversion at tile scales that differ
    by up to 16x, and a reference maximum per row: the first tile's maximum,
    the first tile shifted down by ``ref_drop``, but never more than 8 below
    the row maximum (P' stays under 2^8 <= 448)."""
    rng = np.random.default_rng(seed)
    K = 128 * n_tiles
    x = rng.standard_normal((R, K)) * spread
    x[:, :128] -= ref_drop
    sig = 2.0 ** rng.uniform(-2, 2, n_tiles)
    v = rng.standard_normal((K, D)) * np.repeat(sig, 128)[:, None]
    v = v.astype(np.float32).astype(np.float64)
    sv = np.empty(n_tiles)
    vq = np.empty_like(v)
    for t in range(n_tiles):
        blk = v[128 * t:128 * (t + 1)]
        sv[t] = np.float32(np.abs(blk).max() / 448.0)
        vq[128 * t:128 * (t + 1)] = _e4m3(blk / sv[t]) * sv[t]
    sv_tok = np.repeat(sv, 128)
    vmax = float(sv.max())
    M = x.max(axis=1, keepdims=True)
    m_ref = np.maximum(x[:, :128].max(axis=1, keepdims=True), M - 8.0)
    return x, vq, sv_tok, vmax, M, m_ref


def _emulate(x, vq, sv_tok, vmax, m_ref, sv_used=None, drop_tile=None):
    """An fp8 path's arithmetic: P' = 2^(x - m_ref) sv / vmax rounded to e4m3,
    O = sum P~' code (codes = v / sv), divided by the unrounded sum of
    2^(x - m_ref), times vmax, rounded to bf16.  ``sv_used`` / ``drop_tile``
    plant a mistake (a wrong V block scale; one tile left out of O)."""
    svu = sv_tok if sv_used is None else sv_used
    p = np.exp2(x - m_ref)
    pq = _e4m3(p * svu[None, :] / vmax)
    codes = vq / sv_tok[:, None]
    if drop_tile is not None:
        pq[:, 128 * drop_tile:128 * (drop_tile + 1)] = 0
    o = (pq @ codes) * vmax / p.sum(axis=1, keepdims=True)
    return _bf16(o)


@pytest.mark.parametrize("seed,spread,ref_drop", [
    (1, 1.0, 0.0),     # flat rows: many comparable weights
    (2, 4.0, 0.0),     # peaked rows
    (3, 8.0, 0.0),     # very peaked: most weights in or below e4m3's subnormal range
    (4, 2.0, 6.0),     # the reference maximum far below the row's
    (5, 6.0, 20.0),    # reference 8 below the maximum, large dynamic range
])
def test_p_rounding_model_bounds_an_explicit_e4m3_rounding(seed, spread, ref_drop):
    x, vq, sv_tok, vmax, M, m_ref = _row_case(seed, spread, ref_drop)
    e = np.exp2(x - M)
    o, bound, sigma = fp8.p_rounding_model(e, vq, sv_tok, vmax)
    np.testing.assert_allclose(o, (e @ vq) / e.sum(axis=1, keepdims=True), rtol=1e-12, atol=1e-15)
    got = _emulate(x, vq, sv_tok, vmax, m_ref)
    err = np.abs(got - o)
    assert (err <= bound).all(), float((err / bound).max())
    ratio = float(np.mean((err / sigma) ** 2))
    assert ratio <= 1.0, ratio
    assert err.max() > 0


@pytest.mark.parametrize("mistake", ["v_scale", "drop_tile"])
def test_p_rounding_model_catches_planted_mistakes(mistake):
    # the same rows as the flat case; one wrong V block scale, or one tile of
    # keys missing from P V, must show far above the error scale
    x, vq, sv_tok, vmax, M, m_ref = _row_case(1, 1.0, 0.0)
    e = np.exp2(x - M)
    o, bound, sigma = fp8.p_rounding_model(e, vq, sv_tok, vmax)
    if mistake == "v_scale":
        sv_used = sv_tok.copy()
        sv_used[3 * 128:4 * 128] *= 2
        got = _emulate(x, vq, sv_tok, vmax, m_ref, sv_used=sv_used)
    else:
        got = _emulate(x, vq, sv_tok, vmax, m_ref, drop_tile=5)
    ratio = float(np.mean((np.abs(got - o) / sigma) ** 2))
    assert ratio > 10.0, ratio


def test_fp8_oracle_equals_the_plain_one_on_exactly_representable_operands():
    # Every 128-row block of q, k and v holds e4m3 values times 2^-4 with
    # its largest magnitude exactly 448 * 2^-4: the quantisation is then
    # lossless (scale 2^-4, codes the values themselves), so the fp8 oracle
    # must give the plain oracle's output bit for bit.
    from block_sparse_video_rf_b200 import synth
    w = synth.workload("tiny", N=1, latent=(4, 32, 32), txt_len=0, sparsity=0.5)
    g = oracle.geometry(w.S, w.txt_len, *w.latent)
    rng = np.random.default_rng(7)
    vals = fp8.e4m3_values()
    finite = vals[np.isfinite(vals) & (np.abs(vals) <= 240)]

    def tensor():
        x = rng.choice(finite, size=(w.S, w.D)) * 2.0 ** -4
        for rows in fp8.internal_tiles(g):
            r = rows[rows >= 0]
            x[r[0], 0] = 448 * 2.0 ** -4     # every block's amax is exactly 448 * 2^-4
        return x.astype(np.float32)

    q, k, v = tensor()[None], tensor()[None], tensor()[None]          # BSND with one head: [1, S, 1, D]
    q, k, v = (a[:, :, None, :] for a in (q[0][None], k[0][None], v[0][None]))
    ref, mask, _, _ = oracle.rf_sparse_attention(q, k, v, "BSND", w.txt_len, w.latent, w.sparsity)
    got, mask8, _, _ = fp8.rf_sparse_attention_fp8(q, k, v, "BSND", w.txt_len, w.latent, w.sparsity)
    np.testing.assert_array_equal(mask, mask8)
    np.testing.assert_array_equal(got, ref)
