"""Parity at the full benchmark shapes, in the launch configuration bench.py
times, on sampled heads and rows the oracle computes one by one.

The mask of each sampled head is compared bit for bit (near-ties excused);
output rows are compared within max-abs 2e-2 / mean-abs 2e-3 (bf16, fp16),
or against the oracle over the dequantised operands within the error model of
the e4m3 rounding of P (``parity_util.assert_close_fp8``).  Sampled rows cover text rows, promoted rows,
the partial prefix tile, first-frame blocks and sparse blocks."""

import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_close, assert_close_fp8, fp8_reference, mask_mismatch, unpack_mask

pytestmark = pytest.mark.gpu


def _run(name, dtype=torch.bfloat16, precision="native", **over):
    from block_sparse_video_rf_b200 import rfsa, synth
    w = synth.workload(name, **over)
    q, k, v = synth.make_inputs(w, device="cuda", dtype=dtype)
    sp = np.float32(w.sparsity)
    ws = rfsa.alloc_workspace(w.B, w.S, w.N, w.D, w.txt_len, w.latent, precision=precision)
    out = torch.empty_like(q)
    rfsa.rf_prepare(q, k, v, w.layout, w.txt_len, w.latent, sp, ws, precision=precision)
    rfsa.rf_attend(out, w.layout, w.txt_len, w.latent, sp, ws, precision=precision)
    plan = rfsa.rf_plan(w.S, w.txt_len, w.latent, sp)
    assert rfsa.rf_read_status(ws, w.B, w.N, 128, plan) == 0
    views = rfsa.workspace_views(ws, w.B, w.N, plan, dtype=dtype, precision=precision)
    return w, q, k, v, out, plan, views


def _head(x, n):
    return x[0, :, n].float().cpu().numpy()     # BSND -> [S, D]


def _sample_rows(g, rng, per_kind=6):
    rows = []
    rows += list(rng.choice(np.arange(g.txt_len), min(per_kind, g.txt_len), replace=False)) if g.txt_len else []
    if len(g.promoted):
        rows += list(rng.choice(g.promoted, per_kind, replace=False))
    rows += list(g.prefix[-3:])                                   # last rows of the (partial) prefix tile
    if not g.dense:
        rows += list(g.blocks[0][rng.choice(128, 3, replace=False)])            # first-frame block
        for blk in rng.choice(np.arange(g.ff, g.nb), per_kind, replace=False):
            rows.append(g.blocks[blk][rng.integers(128)])
    return np.array(sorted(set(int(r) for r in rows)))


@pytest.mark.parametrize("name,over,heads", [
    ("minimax", {}, (0, 27, 55)),
    ("minimax", {"sparsity": 0.5}, (3,)),
    ("minimax", {"sparsity": 0.9}, (11,)),
    ("minimax", {"sparsity": 0.0}, (40,)),
    ("wan", {}, (0, 39)),
    ("minimax", {"dtype": torch.float16}, (7,)),
    ("minimax", {"precision": "fp8"}, (5, 50)),
    # the largest block count the library takes: 4096 sparse blocks (524,288 video tokens), one head
    ("tiny", {"N": 1, "latent": (128, 64, 64), "txt_len": 0, "sparsity": 0.5, "seed": 43}, (0,)),
    ("tiny", {"N": 1, "latent": (128, 64, 64), "txt_len": 0, "sparsity": 0.5, "seed": 44, "precision": "fp8"}, (0,)),
])
def test_full_size_sampled(name, over, heads):
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    over = dict(over)
    precision = over.get("precision", "native")
    w, q, k, v, out, plan, views = _run(name, **over)
    g = oracle.geometry(w.S, w.txt_len, *w.latent)
    assert plan.nb == g.nb and plan.P == len(g.prefix)
    rng = np.random.default_rng(123)
    words = views["mask"].cpu().numpy().view(np.uint32)
    scale = w.D ** -0.5
    for n in heads:
        qh, kh, vh = _head(q, n), _head(k, n), _head(v, n)
        mask, margin = oracle.build_mask(qh[None, None], kh[None, None], g, float(np.float32(w.sparsity)))
        bad, excused, near = mask_mismatch(words[0, n][None, None], mask, margin)
        assert bad == 0, f"head {n}: {bad} mask rows differ outside near-ties ({excused} excused, {near} near-ties)"
        gpu_mask = unpack_mask(words[0, n], g.nb)
        rows = _sample_rows(g, rng)
        got = out[0, torch.from_numpy(rows).cuda(), n].float().cpu().numpy()
        if precision == "fp8":
            ref, bound, sigma = fp8_reference(qh, kh, vh, g, gpu_mask, scale, rows=rows)
            assert_close_fp8(got, ref, bound, sigma, f"{name} fp8 head {n}")
        else:
            ref = oracle.attention_rows(qh, kh, vh, g, gpu_mask, scale, rows=rows)
            assert_close(got, ref, f"{name} head {n}")


def _whole_heads(name, heads, **over):
    """Full-size call in the bench's launch configuration; every output row
    of the given heads against the oracle under the GPU's mask (itself
    compared bit for bit with the oracle's, near-ties excused)."""
    w, q, k, v, out, plan, views = _run(name, **over)
    g = oracle.geometry(w.S, w.txt_len, *w.latent)
    words = views["mask"].cpu().numpy().view(np.uint32)
    worst = (0.0, 0.0)
    for n in heads:
        qh, kh, vh = _head(q, n), _head(k, n), _head(v, n)
        if not g.dense:
            mask, margin = oracle.build_mask(qh[None, None], kh[None, None], g, float(np.float32(w.sparsity)))
            bad, excused, near = mask_mismatch(words[0, n][None, None], mask, margin)
            assert bad == 0, f"head {n}: {bad} mask rows differ outside near-ties ({excused} excused)"
        gpu_mask = None if g.dense else unpack_mask(words[0, n], g.nb)
        ref = oracle.attention_rows(qh, kh, vh, g, gpu_mask, w.D ** -0.5)
        got = _head(out, n)
        mx, mean = assert_close(got, ref, f"{name} head {n}, all {w.S} rows")
        worst = (max(worst[0], mx), max(worst[1], mean))
    print(f"{name} heads {heads}: every row, max-abs {worst[0]:.2e} mean-abs {worst[1]:.2e}")


def test_whole_head_minimax():
    # MiniMax-H3 (56 heads, s = 0.8, bf16): all 62,752 rows of head 0
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    _whole_heads("minimax", (0,))


def test_whole_head_wan():
    # the Wan2.2-sized clip (40 heads, latent (21, 45, 80), promotion): all 75,600 rows of head 17
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    _whole_heads("wan", (17,))


def test_text_prefixed_clip_all_heads():
    # the text-prefixed clip at its full 12 heads: every row of every head
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    _whole_heads("text", tuple(range(12)))


def test_half_head_minimax_fp8():
    # fp8 e4m3 at MiniMax-H3: every second row of one head (31,376 rows: text,
    # promoted, first-frame and sparse rows alike) against the oracle over the
    # dequantised operands, under the error model of P's e4m3 rounding
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    w, q, k, v, out, plan, views = _run("minimax", precision="fp8")
    g = oracle.geometry(w.S, w.txt_len, *w.latent)
    words = views["mask"].cpu().numpy().view(np.uint32)
    n = 31
    rows = np.arange(0, w.S, 2)
    qh, kh, vh = _head(q, n), _head(k, n), _head(v, n)
    ref, bound, sigma = fp8_reference(qh, kh, vh, g, unpack_mask(words[0, n], g.nb), w.D ** -0.5, rows=rows)
    got = out[0, torch.from_numpy(rows).cuda(), n].float().cpu().numpy()
    mx, mean, ratio = assert_close_fp8(got, ref, bound, sigma, f"minimax fp8 head {n}, every second row")
    print(f"minimax fp8 head {n}: {len(rows)} rows, max-abs {mx:.2e} mean-abs {mean:.2e} (err/sigma)^2 {ratio:.3f}")


def test_full_size_bnsd_sampled():
    # the caller's BNSD layout at the full MiniMax-H3 shape (the bench runs BSND)
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    w, q, k, v, out, plan, views = _run("minimax", layout="BNSD")
    g = oracle.geometry(w.S, w.txt_len, *w.latent)
    words = views["mask"].cpu().numpy().view(np.uint32)
    rng = np.random.default_rng(321)
    for n in (2, 44):
        qh, kh, vh = (x[0, n].float().cpu().numpy() for x in (q, k, v))     # BNSD -> [S, D]
        mask, margin = oracle.build_mask(qh[None, None], kh[None, None], g, float(np.float32(w.sparsity)))
        bad, excused, near = mask_mismatch(words[0, n][None, None], mask, margin)
        assert bad == 0, f"head {n}: {bad} mask rows differ outside near-ties"
        rows = _sample_rows(g, rng)
        got = out[0, n, torch.from_numpy(rows).cuda()].float().cpu().numpy()
        ref = oracle.attention_rows(qh, kh, vh, g, unpack_mask(words[0, n], g.nb), w.D ** -0.5, rows=rows)
        assert_close(got, ref, f"minimax BNSD head {n}")
