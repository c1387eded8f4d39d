"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Inputs are the seeded bf16 tensors of ``block_sparse_video_rf_b200.synth``;
the oracle gets the same bf16 values widened.  Index work (reorder, mask) is
compared bit for bit (mask rows whose k-th/(k+1)-th block scores are within
1e-5 relative are counted and excused); outputs within max-abs 2e-2 and
mean-abs 2e-3.
"""

import numpy as np
import pytest
import torch

import oracle
from parity_util import (MAX_ABS, MEAN_ABS, assert_close, internal_order, mask_mismatch, pack_mask, to_bnsd_np,
                         to_np, unpack_mask)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rfsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from block_sparse_video_rf_b200 import rfsa as mod
    return mod


def _inputs(name, device="cuda", **over):
    from block_sparse_video_rf_b200 import synth
    w = synth.workload(name, **over)
    q, k, v = synth.make_inputs(w, device="cpu")
    return w, q.to(device), k.to(device), v.to(device)


# (name, overrides) of small cases: several tiles, ragged prefix, promotion, tail, both layouts
CASES = {
    "tiny": ("tiny", {}),
    "text2": ("text", {"N": 2}),
    "ragged": ("tiny", {"txt_len": 37, "latent": (8, 21, 43), "sparsity": 0.7, "seed": 11}),
    "oddtiles_bnsd": ("tiny", {"txt_len": 19, "latent": (5, 24, 40), "sparsity": 0.6, "layout": "BNSD", "seed": 12}),
    "wan_small": ("wan", {"N": 2, "latent": (4, 45, 40)}),
    "rope_small": ("minimax", {"N": 2, "latent": (6, 24, 42)}),
}


def _run_prepare(rfsa, w, q, k, v):
    ws = rfsa.alloc_workspace(w.B, w.S, w.N, w.D, w.txt_len, w.latent)
    rfsa.rf_prepare(q, k, v, w.layout, w.txt_len, w.latent, np.float32(w.sparsity), ws)
    plan = rfsa.rf_plan(w.S, w.txt_len, w.latent, np.float32(w.sparsity))
    views = rfsa.workspace_views(ws, w.B, w.N, plan)
    return ws, plan, views


def _oracle_mask(w, q, k):
    g = oracle.geometry(w.S, w.txt_len, *w.latent)
    qb, kb = to_bnsd_np(q, w.layout), to_bnsd_np(k, w.layout)
    mask, margin = oracle.build_mask(qb, kb, g, float(np.float32(w.sparsity)))
    return g, mask, margin


@pytest.mark.parametrize("case", list(CASES))
def test_reorder_is_bit_exact(rfsa, case):
    name, over = CASES[case]
    w, q, k, v = _inputs(name, **over)
    ws, plan, views = _run_prepare(rfsa, w, q, k, v)
    torch.cuda.synchronize()
    g = oracle.geometry(w.S, w.txt_len, *w.latent)
    order = internal_order(g)
    assert len(order) == plan.S_int
    for src, name_int in ((q, "q_int"), (k, "k_int"), (v, "v_int")):
        exp = torch.zeros((w.B, w.N, plan.S_int, 128), dtype=torch.bfloat16)
        s_bnsd = src.cpu() if w.layout == "BNSD" else src.cpu().transpose(1, 2)
        valid = order >= 0
        exp[:, :, torch.from_numpy(np.nonzero(valid)[0])] = s_bnsd[:, :, torch.from_numpy(order[valid])]
        got = views[name_int].cpu()
        assert torch.equal(got.view(torch.int16), exp.view(torch.int16)), name_int


@pytest.mark.parametrize("case", list(CASES))
def test_pooling_and_mask(rfsa, case):
    name, over = CASES[case]
    w, q, k, v = _inputs(name, **over)
    ws, plan, views = _run_prepare(rfsa, w, q, k, v)
    torch.cuda.synchronize()
    g, mask, margin = _oracle_mask(w, q, k)
    if g.dense:
        return
    qb = to_bnsd_np(q, w.layout)
    for b in range(w.B):
        for n in range(w.N):
            ref = oracle.pool_blocks(qb[b, n], g.blocks)
            np.testing.assert_allclose(to_np(views["pooled_q"][b, n]), ref, rtol=0, atol=2e-6)
    words = views["mask"].cpu().numpy().view(np.uint32)
    bad, excused, near = mask_mismatch(words, mask, margin)
    assert bad == 0, f"{bad} mask rows differ outside near-ties"
    kept = views["kept"].cpu().numpy()
    np.testing.assert_array_equal(kept, unpack_mask(words, g.nb).sum(-1))
    # margins agree where both are finite and not near-ties
    gm = views["margin"].cpu().numpy()
    fin = np.isfinite(margin)
    assert (np.isfinite(gm) == fin).all()
    np.testing.assert_allclose(gm[fin], margin[fin], rtol=1e-3, atol=2e-5)
    print(f"{case}: near-ties {near}, excused mismatching rows {excused}")


@pytest.mark.parametrize("case", list(CASES))
def test_attention_under_oracle_mask(rfsa, case):
    name, over = CASES[case]
    w, q, k, v = _inputs(name, **over)
    ws, plan, views = _run_prepare(rfsa, w, q, k, v)
    g, mask, margin = _oracle_mask(w, q, k)
    if not g.dense:
        views["mask"].copy_(torch.from_numpy(pack_mask(mask).view(np.int32)).cuda())
    out = torch.empty_like(q)
    rfsa.rf_attend(out, w.layout, w.txt_len, w.latent, np.float32(w.sparsity), ws)
    assert rfsa.rf_read_status(ws, w.B, w.N, 128, plan) == 0
    qb, kb, vb = (to_bnsd_np(t, w.layout) for t in (q, k, v))
    scale = w.D ** -0.5
    got = to_bnsd_np(out, w.layout)
    for b in range(w.B):
        for n in range(w.N):
            ref = oracle.attention_rows(qb[b, n], kb[b, n], vb[b, n], g, None if g.dense else mask[b, n], scale)
            assert_close(got[b, n], ref, f"{case} b{b} n{n}")


@pytest.mark.parametrize("case", ["tiny", "ragged", "oddtiles_bnsd"])
def test_end_to_end(rfsa, case):
    name, over = CASES[case]
    w, q, k, v = _inputs(name, **over)
    out = rfsa.rf_sparse_attention(q, k, v, w.layout, w.txt_len, w.latent, np.float32(w.sparsity))
    torch.cuda.synchronize()
    ref, _, _, _ = oracle.rf_sparse_attention(to_np(q), to_np(k), to_np(v), w.layout, w.txt_len, w.latent,
                                              float(np.float32(w.sparsity)))
    assert out.shape == q.shape
    assert_close(to_np(out), ref, case)


def test_sparsity_zero_is_dense_attention(rfsa):
    w, q, k, v = _inputs("tiny", sparsity=0.0, txt_len=40, latent=(2, 32, 64), N=1)
    out = rfsa.rf_sparse_attention(q, k, v, w.layout, w.txt_len, w.latent, 0.0)
    torch.cuda.synchronize()
    qb, kb, vb = (to_bnsd_np(t, w.layout) for t in (q, k, v))
    ref = oracle.dense_attention(qb[0, 0], kb[0, 0], vb[0, 0], w.D ** -0.5)
    assert_close(to_bnsd_np(out, w.layout)[0, 0], ref, "s=0")


def test_page_example_single_frame(rfsa):
    # lite_boost example: B=1, N=3, S=4096, D=128, BSND, latent (1, 64, 64), sparsity 0 -> shape (1, 4096, 3, 128)
    w, q, k, v = _inputs("tiny", N=3, latent=(1, 64, 64), sparsity=0.0, seed=21)
    out = rfsa.rf_sparse_attention(q, k, v, "BSND", 0, (1, 64, 64), 0.0, scale=128 ** -0.5)
    torch.cuda.synchronize()
    assert tuple(out.shape) == (1, 4096, 3, 128)
    qb, kb, vb = (to_bnsd_np(t, "BSND") for t in (q, k, v))
    for n in range(3):
        assert_close(to_bnsd_np(out, "BSND")[0, n], oracle.dense_attention(qb[0, n], kb[0, n], vb[0, n], 128 ** -0.5))


@pytest.mark.parametrize("latent,txt", [((3, 16, 16), 7), ((0, 0, 0), 0)])
def test_dense_fallbacks(rfsa, latent, txt):
    S = txt + latent[0] * latent[1] * latent[2] if latent[0] else 1000
    w, q, k, v = _inputs("tiny", N=2, latent=latent, txt_len=txt, sparsity=0.9, seed=22) if latent[0] else (None,) * 4
    if w is None:
        g = torch.Generator().manual_seed(5)
        q, k, v = (torch.randn((1, S, 2, 128), generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    out = rfsa.rf_sparse_attention(q, k, v, "BSND", txt, latent, 0.9)
    torch.cuda.synchronize()
    qb, kb, vb = (to_bnsd_np(t, "BSND") for t in (q, k, v))
    for n in range(2):
        assert_close(to_bnsd_np(out, "BSND")[0, n], oracle.dense_attention(qb[0, n], kb[0, n], vb[0, n], 128 ** -0.5))


@pytest.mark.parametrize("layout", ["BSND", "BNSD"])
def test_unpermute_inverts_reorder(rfsa, layout):
    w, q, k, v = _inputs("tiny", txt_len=37, latent=(8, 21, 43), layout=layout, seed=13)
    ws, plan, views = _run_prepare(rfsa, w, q, k, v)
    back = torch.zeros_like(q)
    rfsa.rf_unpermute(views["q_int"], back, layout, w.txt_len, w.latent)
    torch.cuda.synchronize()
    assert torch.equal(back.view(torch.int16), q.view(torch.int16))


def test_layouts_agree(rfsa):
    w, q, k, v = _inputs("tiny", seed=14)
    out_s = rfsa.rf_sparse_attention(q, k, v, "BSND", 0, w.latent, 0.5)
    qn, kn, vn = (t.transpose(1, 2).contiguous() for t in (q, k, v))
    out_n = rfsa.rf_sparse_attention(qn, kn, vn, "BNSD", 0, w.latent, 0.5)
    torch.cuda.synchronize()
    assert torch.equal(out_s.transpose(1, 2).contiguous().view(torch.int16), out_n.view(torch.int16))


def test_repeat_calls_are_deterministic(rfsa):
    w, q, k, v = _inputs("text", N=2)
    a = rfsa.rf_sparse_attention(q, k, v, w.layout, w.txt_len, w.latent, 0.8)
    b = rfsa.rf_sparse_attention(q, k, v, w.layout, w.txt_len, w.latent, 0.8)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("precision", ["native", "fp8"])
def test_running_max_that_grows_after_the_first_tile(rfsa, precision):
    # The text prefix tile comes first and holds small scores; the video keys are
    # scaled up, so later tiles exceed the first tile's maximum by far and the
    # kernel must raise its running max (and rescale O and l) mid-row.
    from parity_util import assert_close_fp8, fp8_reference
    w, q, k, v = _inputs("tiny", txt_len=128, latent=(4, 32, 32), N=2, seed=31)
    k = k.clone()
    k[:, w.txt_len:] *= 6.0
    out = rfsa.rf_sparse_attention(q, k, v, w.layout, w.txt_len, w.latent, np.float32(w.sparsity),
                                   precision=precision)
    torch.cuda.synchronize()
    if precision == "native":
        ref, _, _, _ = oracle.rf_sparse_attention(to_np(q), to_np(k), to_np(v), w.layout, w.txt_len, w.latent,
                                                  float(np.float32(w.sparsity)))
        assert_close(to_np(out), ref, "growing max")
    else:
        qb, kb, vb = (to_bnsd_np(t, w.layout) for t in (q, k, v))
        g = oracle.geometry(w.S, w.txt_len, *w.latent)
        mask, _ = oracle.build_mask(qb, kb, g, float(np.float32(w.sparsity)))
        for n in range(w.N):
            ref, bound, sigma = fp8_reference(qb[0, n], kb[0, n], vb[0, n], g, mask[0, n], w.D ** -0.5)
            assert_close_fp8(to_bnsd_np(out, w.layout)[0, n], ref, bound, sigma, f"growing max fp8 n{n}")


@pytest.mark.parametrize("layout", ["BSND", "BNSD"])
def test_batch_of_two(rfsa, layout):
    # B = 2: every (b, head) has its own mask and work units; the permutation is shared
    w, q, k, v = _inputs("tiny", B=2, N=2, txt_len=37, latent=(6, 24, 40), sparsity=0.6, layout=layout, seed=41)
    ws, plan, views = _run_prepare(rfsa, w, q, k, v)
    g, mask, margin = _oracle_mask(w, q, k)
    bad, excused, near = mask_mismatch(views["mask"].cpu().numpy().view(np.uint32), mask, margin)
    assert bad == 0
    out = torch.empty_like(q)
    views["mask"].copy_(torch.from_numpy(pack_mask(mask).view(np.int32)).cuda())
    rfsa.rf_attend(out, w.layout, w.txt_len, w.latent, np.float32(w.sparsity), ws)
    assert rfsa.rf_read_status(ws, w.B, w.N, 128, plan) == 0
    qb, kb, vb = (to_bnsd_np(t, w.layout) for t in (q, k, v))
    got = to_bnsd_np(out, w.layout)
    for b in range(2):
        for n in range(2):
            ref = oracle.attention_rows(qb[b, n], kb[b, n], vb[b, n], g, mask[b, n], w.D ** -0.5)
            assert_close(got[b, n], ref, f"B=2 b{b} n{n}")


def test_sparsity_one_keeps_prefix_and_first_frame(rfsa):
    # sparsity 1 keeps no top-k block: sparse rows read the prefix and the forced first-frame blocks only
    w, q, k, v = _inputs("tiny", txt_len=64, latent=(4, 32, 32), sparsity=1.0, N=2, seed=42)
    out = rfsa.rf_sparse_attention(q, k, v, w.layout, w.txt_len, w.latent, 1.0)
    torch.cuda.synchronize()
    ref, mask, _, g = oracle.rf_sparse_attention(to_np(q), to_np(k), to_np(v), w.layout, w.txt_len, w.latent, 1.0)
    assert (mask[0, :, g.ff:].sum(-1) == g.ff).all()
    assert_close(to_np(out), ref, "s=1")


@pytest.mark.parametrize("S", [1, 2, 127, 129])
def test_tiny_sequences_without_video_geometry(rfsa, S):
    # one query tile with 1..127 valid rows, or a second tile holding one row: a unit of one or two key tiles,
    # the rest of the tile masked
    g = torch.Generator().manual_seed(100 + S)
    q, k, v = (torch.randn((1, S, 3, 128), generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    out = rfsa.rf_sparse_attention(q, k, v, "BSND", 0, (0, 0, 0), 0.5)
    torch.cuda.synchronize()
    qb, kb, vb = (to_bnsd_np(t, "BSND") for t in (q, k, v))
    for n in range(3):
        assert_close(to_bnsd_np(out, "BSND")[0, n], oracle.dense_attention(qb[0, n], kb[0, n], vb[0, n], 128 ** -0.5))


@pytest.mark.parametrize("layout", ["BSND", "BNSD"])
def test_page_signature_call(rfsa, layout):
    # rfsa.sparse_attention, the page's parameter list: rf_v2 gives the direct
    # call's output bit for bit; sparse_type None is dense attention
    w, q, k, v = _inputs("tiny", txt_len=37, latent=(8, 21, 43), sparsity=0.7, layout=layout, seed=71)
    sp = np.float32(w.sparsity)
    a = rfsa.sparse_attention(q, k, v, head_num=w.N, input_layout=layout, sparse_type="rf_v2", txt_len=w.txt_len,
                              latent_shape_q=list(w.latent), sparsity=sp)
    b = rfsa.rf_sparse_attention(q, k, v, layout, w.txt_len, w.latent, sp)
    d = rfsa.sparse_attention(q, k, v, head_num=w.N, input_layout=layout)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    qb, kb, vb = (to_bnsd_np(t, layout) for t in (q, k, v))
    got = to_bnsd_np(d, layout)
    for n in range(w.N):
        assert_close(got[0, n], oracle.dense_attention(qb[0, n], kb[0, n], vb[0, n], w.D ** -0.5), f"dense n{n}")
