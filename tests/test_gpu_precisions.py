"""Parity of the fp16 and fp8 paths (through the C ABI's _ex entry points)
with the CPU oracle.

fp16: the same checks as bf16 -- reorder bit for bit, the block mask bit for
bit (near-ties excused), outputs within max-abs 2e-2 / mean-abs 2e-3 of the
fp64 oracle on the same fp16 values.

fp8 (oracle/fp8.py, readings R14-R15): the e4m3 codes and the per-block
scales bit for bit against the oracle's quantisation (an fp32 computation
taken in the same precision on both sides); the output against the oracle's
attention over the dequantised Q, K, V: every element within the worst-case
bound of the e4m3 rounding of P (which the oracle does not apply) and the
errors on the scale that rounding predicts (``oracle.fp8.p_rounding_model``,
``parity_util.assert_close_fp8``).
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8
from parity_util import (assert_close, assert_close_fp8, fp8_reference, internal_order, mask_mismatch, pack_mask,
                         to_bnsd_np, to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rfsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from block_sparse_video_rf_b200 import rfsa as mod
    return mod


def _inputs(name, dtype, **over):
    from block_sparse_video_rf_b200 import synth
    w = synth.workload(name, **over)
    q, k, v = synth.make_inputs(w, device="cpu", dtype=dtype)
    return w, q.cuda(), k.cuda(), v.cuda()


CASES = {
    "tiny": ("tiny", {}),
    "text2": ("text", {"N": 2}),
    "ragged": ("tiny", {"txt_len": 37, "latent": (8, 21, 43), "sparsity": 0.7, "seed": 11}),
    "oddtiles_bnsd": ("tiny", {"txt_len": 19, "latent": (5, 24, 40), "sparsity": 0.6, "layout": "BNSD", "seed": 12}),
    "rope_small": ("minimax", {"N": 2, "latent": (6, 24, 42)}),
    "dense_fallback": ("tiny", {"N": 2, "latent": (3, 16, 16), "txt_len": 7, "sparsity": 0.9, "seed": 22}),
}


def _prepare(rfsa, w, q, k, v, precision):
    ws = rfsa.alloc_workspace(w.B, w.S, w.N, w.D, w.txt_len, w.latent, precision=precision)
    rfsa.rf_prepare(q, k, v, w.layout, w.txt_len, w.latent, np.float32(w.sparsity), ws, precision=precision)
    plan = rfsa.rf_plan(w.S, w.txt_len, w.latent, np.float32(w.sparsity))
    views = rfsa.workspace_views(ws, w.B, w.N, plan, dtype=q.dtype, precision=precision)
    return ws, plan, views


def _oracle_mask(w, q, k):
    g = oracle.geometry(w.S, w.txt_len, *w.latent)
    mask, margin = oracle.build_mask(to_bnsd_np(q, w.layout), to_bnsd_np(k, w.layout), g,
                                     float(np.float32(w.sparsity)))
    return g, mask, margin


def _attend_under_oracle_mask(rfsa, w, q, k, v, precision):
    ws, plan, views = _prepare(rfsa, w, q, k, v, precision)
    g, mask, margin = _oracle_mask(w, q, k)
    if not g.dense:
        views["mask"].copy_(torch.from_numpy(pack_mask(mask).view(np.int32)).cuda())
    out = torch.empty_like(q)
    rfsa.rf_attend(out, w.layout, w.txt_len, w.latent, np.float32(w.sparsity), ws, precision=precision)
    assert rfsa.rf_read_status(ws, w.B, w.N, 128, plan) == 0
    return out, g, mask, views


# ---------------------------------------------------------------- fp16

@pytest.mark.parametrize("case", ["tiny", "ragged", "oddtiles_bnsd"])
def test_fp16_reorder_and_mask(rfsa, case):
    name, over = CASES[case]
    w, q, k, v = _inputs(name, torch.float16, **over)
    ws, plan, views = _prepare(rfsa, w, q, k, v, "native")
    torch.cuda.synchronize()
    g, mask, margin = _oracle_mask(w, q, k)
    order = internal_order(g)
    valid = order >= 0
    for src, key in ((q, "q_int"), (k, "k_int"), (v, "v_int")):
        exp = torch.zeros((w.B, w.N, plan.S_int, 128), dtype=torch.float16)
        s_bnsd = src.cpu() if w.layout == "BNSD" else src.cpu().transpose(1, 2)
        exp[:, :, torch.from_numpy(np.nonzero(valid)[0])] = s_bnsd[:, :, torch.from_numpy(order[valid])]
        assert torch.equal(views[key].cpu().view(torch.int16), exp.view(torch.int16)), key
    if not g.dense:
        bad, excused, near = mask_mismatch(views["mask"].cpu().numpy().view(np.uint32), mask, margin)
        assert bad == 0, f"{bad} mask rows differ outside near-ties"


@pytest.mark.parametrize("case", ["tiny", "text2", "ragged", "oddtiles_bnsd", "rope_small", "dense_fallback"])
def test_fp16_attention(rfsa, case):
    name, over = CASES[case]
    w, q, k, v = _inputs(name, torch.float16, **over)
    out, g, mask, _ = _attend_under_oracle_mask(rfsa, w, q, k, v, "native")
    assert out.dtype == torch.float16
    qb, kb, vb = (to_bnsd_np(t, w.layout) for t in (q, k, v))
    got = to_bnsd_np(out, w.layout)
    for b in range(w.B):
        for n in range(w.N):
            ref = oracle.attention_rows(qb[b, n], kb[b, n], vb[b, n], g, None if g.dense else mask[b, n],
                                        w.D ** -0.5)
            mx, mean = assert_close(got[b, n], ref, f"{case} fp16 b{b} n{n}")
    print(f"{case} fp16: max-abs {mx:.2e} mean-abs {mean:.2e}")


def test_fp16_end_to_end_cached_workspace(rfsa):
    w, q, k, v = _inputs("tiny", torch.float16)
    out = rfsa.rf_sparse_attention(q, k, v, w.layout, w.txt_len, w.latent, np.float32(w.sparsity))
    torch.cuda.synchronize()
    ref, _, _, _ = oracle.rf_sparse_attention(to_np(q), to_np(k), to_np(v), w.layout, w.txt_len, w.latent,
                                              float(np.float32(w.sparsity)))
    assert out.dtype == torch.float16
    assert_close(to_np(out), ref, "fp16 e2e")


# ---------------------------------------------------------------- fp8

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("case", ["tiny", "ragged", "oddtiles_bnsd", "dense_fallback"])
def test_fp8_quantisation_is_bit_exact(rfsa, case, dtype):
    name, over = CASES[case]
    w, q, k, v = _inputs(name, dtype, **over)
    ws, plan, views = _prepare(rfsa, w, q, k, v, "fp8")
    torch.cuda.synchronize()
    g = oracle.geometry(w.S, w.txt_len, *w.latent)
    n_tiles = plan.n_tiles
    assert len(fp8.internal_tiles(g)) == n_tiles
    for src, key in ((q, "q"), (k, "k"), (v, "v")):
        xb = to_bnsd_np(src, w.layout)
        got = views[key + "8"].cpu().numpy()
        scales = views[key + "_scales"].cpu().numpy()
        for b in range(w.B):
            for n in range(w.N):
                _, codes, sc = fp8.quantize_head(xb[b, n], g)
                np.testing.assert_array_equal(scales[b, n].view(np.uint32), sc.view(np.uint32))
                if key == "v":
                    np.testing.assert_array_equal(got[b, n], codes.transpose(0, 2, 1))
                else:
                    np.testing.assert_array_equal(got[b, n].reshape(n_tiles, 128, 128), codes)
    np.testing.assert_array_equal(views["vmax"].cpu().numpy(), views["v_scales"].cpu().numpy().max(axis=-1))


CASES["ragged_b2"] = ("tiny", {"B": 2, "N": 2, "txt_len": 37, "latent": (8, 21, 43), "sparsity": 0.7, "seed": 13})
CASES["oddtiles_bnsd_b2"] = ("tiny", {"B": 2, "txt_len": 19, "latent": (5, 24, 40), "sparsity": 0.6,
                                      "layout": "BNSD", "seed": 14})


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("case", ["ragged_b2", "oddtiles_bnsd_b2"])
def test_fp8_quantisation_is_bit_exact_two_batches(rfsa, case, dtype):
    test_fp8_quantisation_is_bit_exact(rfsa, case, dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("case", ["ragged", "ragged_b2", "oddtiles_bnsd_b2", "rope_small"])
def test_fp8_prepare_gives_the_native_mask(rfsa, case, dtype):
    # K1's fp8 form sums the block means in the 16-bit form's order, so the
    # means, and with them the mask, its kept counts and margins, are the
    # native precision's bit for bit
    name, over = CASES[case]
    w, q, k, v = _inputs(name, dtype, **over)
    _, _, nat = _prepare(rfsa, w, q, k, v, "native")
    _, _, f8 = _prepare(rfsa, w, q, k, v, "fp8")
    torch.cuda.synchronize()
    for key in ("pooled_q", "pooled_k", "mask", "kept", "margin"):
        assert torch.equal(nat[key].view(torch.int32), f8[key].view(torch.int32)), key


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("case", ["tiny", "text2", "ragged", "oddtiles_bnsd", "rope_small", "dense_fallback"])
def test_fp8_attention(rfsa, case, dtype):
    name, over = CASES[case]
    w, q, k, v = _inputs(name, dtype, **over)
    out, g, mask, _ = _attend_under_oracle_mask(rfsa, w, q, k, v, "fp8")
    assert out.dtype == dtype
    qb, kb, vb = (to_bnsd_np(t, w.layout) for t in (q, k, v))
    got = to_bnsd_np(out, w.layout).astype(np.float64)
    for b in range(w.B):
        for n in range(w.N):
            ref, bound, sigma = fp8_reference(qb[b, n], kb[b, n], vb[b, n], g, None if g.dense else mask[b, n],
                                              w.D ** -0.5)
            mx, mean, ratio = assert_close_fp8(got[b, n], ref, bound, sigma, f"{case} fp8 b{b} n{n}")
            print(f"{case} fp8 ({dtype}) b{b} n{n}: max-abs {mx:.2e} mean-abs {mean:.2e} (err/sigma)^2 {ratio:.3f}")


def test_fp8_end_to_end_cached_workspace(rfsa):
    w, q, k, v = _inputs("tiny", torch.bfloat16)
    out = rfsa.rf_sparse_attention(q, k, v, w.layout, w.txt_len, w.latent, np.float32(w.sparsity), precision="fp8")
    torch.cuda.synchronize()
    g = oracle.geometry(w.S, w.txt_len, *w.latent)
    qb, kb, vb = (to_bnsd_np(t, w.layout) for t in (q, k, v))
    mask, _ = oracle.build_mask(qb, kb, g, float(np.float32(w.sparsity)))
    got = to_bnsd_np(out, w.layout)
    for n in range(w.N):
        ref, bound, sigma = fp8_reference(qb[0, n], kb[0, n], vb[0, n], g, mask[0, n], w.D ** -0.5)
        assert_close_fp8(got[0, n], ref, bound, sigma, f"fp8 e2e n{n}")


def test_bad_dtype_and_precision_are_rejected(rfsa):
    w, q, k, v = _inputs("tiny", torch.bfloat16)
    with pytest.raises(rfsa.RfError):
        rfsa.rf_sparse_attention(q.float(), k.float(), v.float(), w.layout, 0, w.latent, 0.5)
    with pytest.raises(rfsa.RfError):
        rfsa.rf_sparse_attention(q, k, v, w.layout, 0, w.latent, 0.5, precision="fp4")
