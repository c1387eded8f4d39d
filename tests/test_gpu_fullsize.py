"""Parity at the full benchmark shapes, in the launch configuration bench.py
times, on sampled heads and rows the oracle computes one by one.

The mask of each sampled head is compared bit for bit (near-ties excused);
output rows are compared within max-abs 2e-2 / mean-abs 2e-3 (bf16, fp16),
or against the oracle over the dequantised operands within the fp8 bounds
of ``parity_util.fp8_bounds``.  Sampled rows cover text rows, promoted rows,
the partial prefix tile, first-frame blocks and sparse blocks."""

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8
from parity_util import assert_close, assert_close_fp8, mask_mismatch, unpack_mask

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
            qd, kd, vd = (fp8.quantize_head(x, g)[0] for x in (qh, kh, vh))
            ref = oracle.attention_rows(qd, kd, vd, g, gpu_mask, scale, rows=rows)
            assert_close_fp8(got, ref, vd, f"{name} fp8 head {n}")
        else:
            ref = oracle.attention_rows(qh, kh, vh, g, gpu_mask, scale, rows=rows)
            assert_close(got, ref, f"{name} head {n}")
