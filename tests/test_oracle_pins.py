"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test names what fixes the expected value: a number printed on the pages
(``tests/golden``), a textbook routine (torch's scaled-dot-product attention
in fp64), an exhaustive search on tiny inputs, or an invariant of the
definitions.  None of these calls the CUDA library.
"""

import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import rf_v2


def _sdpa(q, k, v, scale, mask=None):
    """Reference attention from torch (fp64, CPU): [S, D] inputs."""
    t = [torch.from_numpy(np.asarray(a, dtype=np.float64))[None, None] for a in (q, k, v)]
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(*t, attn_mask=m, scale=scale)
    return o[0, 0].numpy()


def _rand(shape, seed):
    g = np.random.default_rng(seed)
    x = g.standard_normal(shape).astype(np.float32)
    # round through bf16 like the real inputs
    return torch.from_numpy(x).to(torch.bfloat16).float().numpy()


# ---------------------------------------------------------------- geometry

def test_worked_geometry_minimax(golden):
    ex = golden["minimax_h3_1344x768"]
    T, H, W = ex["latent"]
    g = oracle.geometry(256 + T * H * W, 256, T, H, W)
    assert T * H * W == ex["video_rows"]
    assert len(g.promoted) + len(g.tail) == ex["promoted_rows"]
    assert g.blocks.size == ex["sparse_rows"]
    assert g.nb == ex["sparse_blocks"]
    assert not g.dense


def test_worked_token_count_single_frame(golden):
    ex = golden["single_frame_64x64"]
    T, H, W = ex["latent"]
    assert T * H * W == ex["tokens"]
    g = oracle.geometry(ex["tokens"], 0, T, H, W)
    assert g.nb == 32 and g.ff == 32          # one frame: every block is a first-frame block


def test_min_sparse_blocks_fallback(golden):
    lim = golden["min_sparse_blocks"]["value"]
    # 31 blocks -> dense; 32 blocks -> sparse path
    g31 = oracle.geometry(31 * 128, 0, 31, 8, 16)
    g32 = oracle.geometry(32 * 128, 0, 32, 8, 16)
    assert g31.dense and not g32.dense and g32.nb == lim


@pytest.mark.parametrize("T,H,W", [(1, 8, 8), (3, 16, 24), (2, 48, 64), (5, 24, 40)])
def test_no_promotion_on_aligned_grid(T, H, W, golden):
    assert golden["aligned_grid_no_promotion"]["tile"] == rf_v2.TILE
    g = oracle.geometry(T * H * W, 0, T, H, W)
    assert len(g.promoted) == 0


@pytest.mark.parametrize("T,H,W", [(62, 24, 42), (21, 45, 80), (3, 13, 29), (2, 7, 100), (4, 9, 9)])
def test_promoted_count(T, H, W):
    g = oracle.geometry(T * H * W, 0, T, H, W)
    Ha, Wa = 8 * (H // 8), 8 * (W // 8)
    assert len(g.promoted) == T * (H * W - Ha * Wa)
    # promoted tokens are exactly those outside the aligned sub-grid
    for s in g.promoted[:200]:
        t, r = divmod(int(s), H * W)
        y, x = divmod(r, W)
        assert y >= Ha or x >= Wa


@pytest.mark.parametrize("txt,T,H,W", [(0, 4, 32, 32), (37, 3, 21, 43), (256, 2, 24, 42), (5, 5, 24, 40)])
def test_partition_is_a_bijection(txt, T, H, W):
    g = oracle.geometry(txt + T * H * W, txt, T, H, W)
    allidx = np.concatenate([g.prefix, g.blocks.ravel()])
    assert np.array_equal(np.sort(allidx), np.arange(txt + T * H * W))
    assert np.array_equal(g.prefix[:txt], np.arange(txt))


@pytest.mark.parametrize("txt,T,H,W", [(0, 4, 32, 32), (11, 3, 24, 42), (0, 21, 45, 80)])
def test_each_block_is_two_whole_tiles(txt, T, H, W):
    # A block holds two whole 8x8 tiles; with an odd tile count per frame the
    # two tiles may come from consecutive frames (as at the (62, 24, 42) grid).
    g = oracle.geometry(txt + T * H * W, txt, T, H, W)
    for blk in g.blocks:
        v = blk - txt
        t, r = np.divmod(v, H * W)
        y, x = np.divmod(r, W)
        tiles = sorted(set(zip(t.tolist(), (y // 8).tolist(), (x // 8).tolist())))
        assert len(tiles) == 2
        assert tiles[1][0] - tiles[0][0] in (0, 1)
        for tt, ty, tx in tiles:
            sel = (t == tt) & (y // 8 == ty) & (x // 8 == tx)
            assert sel.sum() == 64
            assert set(zip((y[sel] % 8).tolist(), (x[sel] % 8).tolist())) == {(a, b) for a in range(8) for b in range(8)}


def test_tile_order_by_enumeration():
    # Nested-loop enumeration of the reading: frames, then 8x8 tiles row-major, then raster inside a tile.
    txt, T, H, W = 3, 2, 19, 35
    g = oracle.geometry(txt + T * H * W, txt, T, H, W)
    Ha, Wa = 8 * (H // 8), 8 * (W // 8)
    seq = []
    for t in range(T):
        for ty in range(Ha // 8):
            for tx in range(Wa // 8):
                for iy in range(8):
                    for ix in range(8):
                        seq.append(txt + t * H * W + (8 * ty + iy) * W + 8 * tx + ix)
    nb = len(seq) // 128
    assert g.nb == nb == 8 and len(seq) == 2 * 16 * 32  # 2 frames x 8 tiles x 64 tokens
    assert g.dense                                   # 8 < 32 blocks: the order is still defined
    assert np.array_equal(g.blocks.ravel(), np.array(seq[: nb * 128]))
    assert np.array_equal(g.tail, np.array(seq[nb * 128:]))


def test_odd_tile_count_promotes_last_half_block():
    # latent (5, 24, 40): 5 * 15 tiles = 75 tiles -> 37 whole blocks + 64 tokens promoted (reading R2)
    g = oracle.geometry(5 * 24 * 40, 0, 5, 24, 40)
    assert g.nb == 37 and len(g.tail) == 64 and len(g.promoted) == 0
    assert len(g.prefix) == 64


@pytest.mark.parametrize("T,H,W", [(62, 24, 42), (4, 32, 32), (8, 48, 64), (21, 45, 80), (2, 40, 24)])
def test_first_frame_blocks(T, H, W):
    g = oracle.geometry(T * H * W, 0, T, H, W)
    Ha, Wa = 8 * (H // 8), 8 * (W // 8)
    assert g.ff == math.ceil(Ha * Wa / 128)
    assert g.first_frame[: g.ff].all() and not g.first_frame[g.ff:].any()


def test_minimax_first_frame_is_eight():
    g = oracle.geometry(256 + 62 * 24 * 42, 256, 62, 24, 42)
    assert g.ff == 8            # 24*40 = 960 aligned tokens per frame = 7.5 blocks


# ---------------------------------------------------------------- kept count

def test_kept_count_fixed_points():
    for nb in (32, 33, 192, 465, 525):
        assert oracle.kept_count(nb, 0.0) == nb        # sparsity 0 disables sparsity
        assert oracle.kept_count(nb, 1.0) == 0
    assert oracle.kept_count(32, 0.5) == 16            # 0.5 prunes half the blocks
    assert oracle.kept_count(192, 0.5) == 96
    # readings (rounding of the dropped count down)
    assert oracle.kept_count(465, 0.8) == 93
    assert oracle.kept_count(192, 0.8) == 39
    assert oracle.kept_count(525, 0.8) == 105
    assert oracle.kept_count(465, 0.9) == 47
    ks = [oracle.kept_count(465, s / 100) for s in range(101)]
    assert all(a >= b for a, b in zip(ks, ks[1:]))


def test_block_means_of_constant_and_index_rows():
    # the mean of a block's 128 rows: rows all equal to c give c; rows equal
    # to their token index give the mean of the block's token indices
    txt, T, H, W = 16, 4, 32, 40
    S = txt + T * H * W
    g = oracle.geometry(S, txt, T, H, W)
    c = np.linspace(-3, 3, 128).astype(np.float32)
    np.testing.assert_array_equal(oracle.pool_blocks(np.tile(c, (S, 1)), g.blocks), np.tile(c, (g.nb, 1)))
    idx = np.tile(np.arange(S, dtype=np.float32)[:, None], (1, 128))
    want = np.array([sum(int(t) for t in blk) / 128.0 for blk in g.blocks], dtype=np.float32)
    np.testing.assert_array_equal(oracle.pool_blocks(idx, g.blocks), np.tile(want[:, None], (1, 128)))


# ---------------------------------------------------------------- top-k

def _brute_topk(row, k):
    """Every k-subset that no swap improves (higher score, or equal score and lower index)."""
    nb = len(row)
    found = []
    for sub in itertools.combinations(range(nb), k):
        s = set(sub)
        ok = all(row[j] > row[jj] or (row[j] == row[jj] and j < jj)
                 for j in s for jj in range(nb) if jj not in s)
        if ok:
            found.append(s)
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("seed", range(12))
def test_topk_matches_exhaustive_search(seed):
    rng = np.random.default_rng(seed)
    nb = int(rng.integers(4, 10))
    scores = rng.integers(-3, 4, size=(nb, nb)).astype(np.float32)   # many exact ties
    ff = np.zeros(nb, bool)
    for k in range(0, nb + 1):
        mask, _ = oracle.topk_mask(scores, k, ff)
        for i in range(nb):
            assert set(np.nonzero(mask[i])[0].tolist()) == _brute_topk(scores[i], k)


def test_topk_first_frame_rows_and_columns():
    rng = np.random.default_rng(7)
    nb, k = 9, 3
    scores = rng.standard_normal((nb, nb)).astype(np.float32)
    ff = np.zeros(nb, bool)
    ff[:2] = True
    mask, margin = oracle.topk_mask(scores, k, ff)
    assert mask[:2].all() and np.isinf(margin[:2]).all()
    for i in range(2, nb):
        expect = _brute_topk(scores[i], k) | {0, 1}
        assert set(np.nonzero(mask[i])[0].tolist()) == expect
        assert k <= mask[i].sum() <= k + 2


def test_margin_value():
    row = np.tile(np.array([5.0, 1.0, 4.0, 2.0], dtype=np.float32), (4, 1))
    _, m = oracle.topk_mask(row, 2, np.zeros(4, bool))
    assert m[0] == pytest.approx((4.0 - 2.0) / 4.0)
    _, m = oracle.topk_mask(row, 4, np.zeros(4, bool))
    assert np.isinf(m[0])
    row[:, 3] = 4.0                                       # exact tie at the boundary
    _, m = oracle.topk_mask(row, 2, np.zeros(4, bool))
    assert m[0] == 0.0


# ---------------------------------------------------------------- attention

def _qkv(S, D, seed):
    return _rand((S, D), seed), _rand((S, D), seed + 1), _rand((S, D), seed + 2)


def test_sparsity_zero_equals_dense_sdpa():
    T, H, W, txt, D = 2, 32, 64, 40, 128
    S = txt + T * H * W
    q, k, v = _qkv(S, D, 10)
    scale = D ** -0.5
    out, mask, _, g = oracle.rf_sparse_attention(q[None, :, None], k[None, :, None], v[None, :, None],
                                                 "BSND", txt, (T, H, W), 0.0)
    assert not g.dense and mask.all()
    ref = _sdpa(q, k, v, scale)
    np.testing.assert_allclose(out[0, :, 0], ref, rtol=0, atol=1e-10)


def test_single_frame_is_dense_for_any_sparsity():
    T, H, W, D = 1, 64, 64, 128
    S = T * H * W
    q, k, v = _qkv(S, D, 20)
    out, _, _, g = oracle.rf_sparse_attention(q[None, None], k[None, None], v[None, None], "BNSD", 0, (T, H, W), 0.8,
                                              scale=0.1)
    assert g.nb == 32 and g.ff == 32
    np.testing.assert_allclose(out[0, 0], _sdpa(q, k, v, 0.1), rtol=0, atol=1e-10)


def test_few_blocks_and_no_geometry_fall_back_to_dense():
    D = 128
    q, k, v = _qkv(3 * 16 * 16 + 7, D, 30)
    out, _, _, g = oracle.rf_sparse_attention(q[None, :, None], k[None, :, None], v[None, :, None], "BSND", 7,
                                              (3, 16, 16), 0.9)
    assert g.dense
    np.testing.assert_allclose(out[0, :, 0], _sdpa(q, k, v, D ** -0.5), rtol=0, atol=1e-10)
    out2, _, _, g2 = oracle.rf_sparse_attention(q[None, :, None], k[None, :, None], v[None, :, None], "BSND", 0,
                                                (0, 0, 0), 0.9)
    assert g2.dense
    np.testing.assert_allclose(out2, out, rtol=0, atol=0)


def _token_mask(g, mask_bn):
    """Boolean [S, S] attend-mask in token order built from the oracle's key sets."""
    m = np.zeros((g.S, g.S), dtype=bool)
    m[g.prefix] = True
    for i in range(g.nb):
        m[np.ix_(g.blocks[i], rf_v2.key_set(g, mask_bn, i))] = True
    return m


def test_masked_attention_matches_sdpa_with_explicit_mask():
    txt, T, H, W, D = 24, 4, 36, 32, 128          # H = 36 promotes 4 rows per frame
    S = txt + T * H * W
    q, k, v = _qkv(S, D, 40)
    out, mask, _, g = oracle.rf_sparse_attention(q[None, :, None], k[None, :, None], v[None, :, None],
                                                 "BSND", txt, (T, H, W), 0.5)
    assert not g.dense and g.nb == 32
    tm = _token_mask(g, mask[0, 0])
    assert 0.3 < tm.mean() < 0.9
    np.testing.assert_allclose(out[0, :, 0], _sdpa(q, k, v, D ** -0.5, tm), rtol=0, atol=1e-10)
    # prefix rows are plain dense rows
    ref = _sdpa(q, k, v, D ** -0.5)
    np.testing.assert_allclose(out[0, g.prefix, 0], ref[g.prefix], rtol=0, atol=1e-10)


def test_one_hot_value_probe_reads_exactly_the_expected_blocks():
    """Engineered scores: s_ij = +/- w_j, so the kept set is known without the oracle's top-k.

    V carries the block id as a one-hot channel, so the support of an output
    row is the set of blocks the row attends to.
    """
    txt, T, H, W, D = 16, 4, 32, 32, 128
    S = txt + T * H * W
    g = oracle.geometry(S, txt, T, H, W)
    nb, ff = g.nb, g.ff
    assert nb == 32 and ff == 8
    rng = np.random.default_rng(3)
    w = rng.permutation(nb).astype(np.float32) / 8.0 + 0.25          # distinct positive weights
    q = np.zeros((S, D), np.float32)
    k = np.zeros((S, D), np.float32)
    v = np.zeros((S, D), np.float32)
    sign = np.ones(nb, np.float32)
    sign[1::2] = -1.0
    for j in range(nb):
        k[g.blocks[j], 0] = w[j]
        q[g.blocks[j], 0] = sign[j]
        v[g.blocks[j], j] = 1.0
    q[g.prefix, 0] = 1.0
    v[g.prefix, 127] = 1.0
    kk = oracle.kept_count(nb, 0.75)
    out, mask, _, _ = oracle.rf_sparse_attention(q[None, :, None], k[None, :, None], v[None, :, None],
                                                 "BSND", txt, (T, H, W), 0.75)
    top = set(np.argsort(-w)[:kk].tolist())
    bottom = set(np.argsort(w)[:kk].tolist())
    for i in range(nb):
        if i < ff:
            expect = set(range(nb))
        else:
            expect = (top if sign[i] > 0 else bottom) | set(range(ff))
        row = out[0, g.blocks[i][5], 0]
        support = set(np.nonzero(row[:nb] > 0)[0].tolist())
        assert support == expect, i
        assert row[127] > 0                                  # prefix always read
        assert set(np.nonzero(mask[0, 0, i])[0].tolist()) == expect


def test_constant_value_gives_constant_output():
    txt, T, H, W, D = 8, 4, 32, 40, 128
    S = txt + T * H * W
    q, k, _ = _qkv(S, D, 50)
    c = np.linspace(-1, 1, D).astype(np.float32)
    v = np.tile(c, (S, 1))
    out, _, _, _ = oracle.rf_sparse_attention(q[None, :, None], k[None, :, None], v[None, :, None],
                                              "BSND", txt, (T, H, W), 0.9)
    np.testing.assert_allclose(out[0, :, 0], np.tile(c, (S, 1)), rtol=0, atol=1e-12)


def test_layouts_agree_and_mask_ignores_query_scale():
    txt, T, H, W, D, N = 0, 4, 32, 32, 128, 2
    S = txt + T * H * W
    rng_q = _rand((1, N, S, D), 60)
    rng_k = _rand((1, N, S, D), 61)
    rng_v = _rand((1, N, S, D), 62)
    o1, m1, _, _ = oracle.rf_sparse_attention(rng_q, rng_k, rng_v, "BNSD", txt, (T, H, W), 0.5)
    t = lambda a: np.ascontiguousarray(np.transpose(a, (0, 2, 1, 3)))
    o2, m2, _, _ = oracle.rf_sparse_attention(t(rng_q), t(rng_k), t(rng_v), "BSND", txt, (T, H, W), 0.5)
    np.testing.assert_array_equal(m1, m2)
    np.testing.assert_allclose(t(o1), o2, rtol=0, atol=0)
    _, m3, _, _ = oracle.rf_sparse_attention(rng_q * 4.0, rng_k, rng_v, "BNSD", txt, (T, H, W), 0.5)
    np.testing.assert_array_equal(m1, m3)
    kk = oracle.kept_count(32, 0.5)
    cnt = m1.sum(-1)[..., 8:]
    assert (cnt >= kk).all() and (cnt <= kk + 8).all()


def test_sparsity_range_is_checked():
    q = np.zeros((1, 4096, 1, 128), np.float32)
    for s in (-0.1, 1.1, float("nan"), float("inf")):
        with pytest.raises(ValueError):
            oracle.rf_sparse_attention(q, q, q, "BSND", 0, (4, 32, 32), s)
    with pytest.raises(ValueError):
        oracle.to_bnsd(q, "SBND")


# ---------------------------------------------------------------- a key geometry of its own (R17)

def test_key_geometry_equal_to_query_changes_nothing():
    txt, T, H, W, D = 16, 4, 32, 40, 128
    S = txt + T * H * W
    q, k, v = _qkv(S, D, 60)
    a, ma, _, _ = oracle.rf_sparse_attention(q[None, :, None], k[None, :, None], v[None, :, None], "BSND", txt,
                                             (T, H, W), 0.6)
    b, mb, _, _ = oracle.rf_sparse_attention(q[None, :, None], k[None, :, None], v[None, :, None], "BSND", txt,
                                             (T, H, W), 0.6, latent_k=(T, H, W))
    np.testing.assert_array_equal(ma, mb)
    np.testing.assert_array_equal(a, b)


def test_key_geometry_sparsity_zero_is_rectangular_sdpa():
    txt, D = 40, 128
    Sq, Sk = txt + 2 * 32 * 64, txt + 3 * 32 * 48
    q = _rand((Sq, D), 61)
    k, v = _rand((Sk, D), 62), _rand((Sk, D), 63)
    out, mask, _, (gq, gk) = oracle.rf_sparse_attention(q[None, :, None], k[None, :, None], v[None, :, None], "BSND",
                                                        txt, (2, 32, 64), 0.0, latent_k=(3, 32, 48))
    assert not gq.dense and not gk.dense and mask.shape == (1, 1, gq.nb, gk.nb) and mask.all()
    np.testing.assert_allclose(out[0, :, 0], _sdpa(q, k, v, D ** -0.5), rtol=0, atol=1e-10)


def test_key_geometry_either_side_dense_is_dense():
    txt, D = 7, 128
    Sq, Sk = txt + 3 * 16 * 16, txt + 4 * 32 * 32        # the query side has 6 blocks: dense
    q = _rand((Sq, D), 64)
    k, v = _rand((Sk, D), 65), _rand((Sk, D), 66)
    out, _, _, (gq, gk) = oracle.rf_sparse_attention(q[None, :, None], k[None, :, None], v[None, :, None], "BSND",
                                                     txt, (3, 16, 16), 0.9, latent_k=(4, 32, 32))
    assert gq.dense and not gk.dense
    np.testing.assert_allclose(out[0, :, 0], _sdpa(q, k, v, D ** -0.5), rtol=0, atol=1e-10)


@pytest.mark.parametrize("seed", range(6))
def test_rectangular_topk_matches_exhaustive_search(seed):
    rng = np.random.default_rng(100 + seed)
    nbq, nbk = int(rng.integers(3, 7)), int(rng.integers(5, 10))
    scores = rng.integers(-3, 4, size=(nbq, nbk)).astype(np.float32)
    ffq = np.zeros(nbq, bool)
    ffq[0] = True
    ffk = np.zeros(nbk, bool)
    ffk[:2] = True
    for k in range(0, nbk + 1):
        mask, _ = oracle.topk_mask(scores, k, ffq, ffk)
        assert mask.shape == (nbq, nbk) and mask[0].all()
        for i in range(1, nbq):
            assert set(np.nonzero(mask[i])[0].tolist()) == _brute_topk(scores[i], k) | {0, 1}


def test_key_geometry_one_hot_value_probe():
    """As the square probe, with query blocks from one grid and key blocks from another."""
    txt, D = 16, 128
    lq, lk = (4, 32, 32), (5, 32, 40)
    Sq, Sk = txt + 4 * 32 * 32, txt + 5 * 32 * 40
    gq, gk = oracle.geometry(Sq, txt, *lq), oracle.geometry(Sk, txt, *lk)
    assert gq.nb == 32 and gk.nb == 50 and gq.ff == 8 and gk.ff == 10
    rng = np.random.default_rng(5)
    w = rng.permutation(gk.nb).astype(np.float32) / 8.0 + 0.25
    q = np.zeros((Sq, D), np.float32)
    k = np.zeros((Sk, D), np.float32)
    v = np.zeros((Sk, D), np.float32)
    sign = np.ones(gq.nb, np.float32)
    sign[1::2] = -1.0
    for j in range(gk.nb):
        k[gk.blocks[j], 0] = w[j]
        v[gk.blocks[j], j] = 1.0
    for i in range(gq.nb):
        q[gq.blocks[i], 0] = sign[i]
    q[gq.prefix, 0] = 1.0
    v[gk.prefix, 127] = 1.0
    kk = oracle.kept_count(gk.nb, 0.7)
    out, mask, _, _ = oracle.rf_sparse_attention(q[None, :, None], k[None, :, None], v[None, :, None], "BSND",
                                                 txt, lq, 0.7, latent_k=lk)
    top = set(np.argsort(-w)[:kk].tolist())
    bottom = set(np.argsort(w)[:kk].tolist())
    for i in range(gq.nb):
        expect = set(range(gk.nb)) if i < gq.ff else (top if sign[i] > 0 else bottom) | set(range(gk.ff))
        row = out[0, gq.blocks[i][3], 0]
        assert set(np.nonzero(row[:gk.nb] > 0)[0].tolist()) == expect, i
        assert row[127] > 0
        assert set(np.nonzero(mask[0, 0, i])[0].tolist()) == expect
