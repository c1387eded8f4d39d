"""Parity of calls whose keys and values have a geometry of their own
(lite_boost.ops.sparse_attention, latent_shape_k; oracle reading R17) with the
CPU oracle: the rectangular block mask bit for bit (near-ties excused), the
output within max-abs 2e-2 / mean-abs 2e-3 (bf16, fp16) or the fp8 bounds,
the fp8 codes and scales of each side bit for bit."""

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8
from parity_util import (assert_close, assert_close_fp8, fp8_reference, mask_mismatch, pack_mask, to_bnsd_np,
                         to_np)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rfsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from block_sparse_video_rf_b200 import rfsa as mod
    return mod


# (query latent, key/value latent, txt_len, sparsity, layout, heads)
CASES = {
    "longer_kv": ((4, 32, 32), (5, 32, 40), 16, 0.7, "BSND", 2),
    "shorter_kv_promoted": ((8, 24, 40), (5, 29, 43), 37, 0.6, "BNSD", 2),
    "odd_tiles_q": ((5, 24, 40), (4, 32, 48), 19, 0.8, "BSND", 1),
    "query_side_dense": ((3, 16, 16), (4, 32, 32), 7, 0.9, "BSND", 2),
    "kv_without_geometry": ((4, 32, 32), (0, 0, 0), 16, 0.5, "BSND", 1),
}


def _inputs(case, dtype=torch.bfloat16):
    from block_sparse_video_rf_b200 import synth
    lq, lk, txt, sp, layout, N = CASES[case]
    wq = synth.workload("tiny", N=N, latent=lq, txt_len=txt, sparsity=sp, layout=layout, seed=61)
    Sk = txt + lk[0] * lk[1] * lk[2] if lk[0] else 3000
    wk = synth.workload("tiny", N=N, latent=lk if lk[0] else (1, 1, Sk - txt), txt_len=txt, layout=layout, seed=62)
    q, _, _ = synth.make_inputs(wq, device="cpu", dtype=dtype)
    _, k, v = synth.make_inputs(wk, device="cpu", dtype=dtype)
    return wq, lk, Sk, q.cuda(), k.cuda(), v.cuda()


def _plans(rfsa, w, lk, Sk):
    return rfsa.rf_plan_kv(w.S, w.txt_len, w.latent, Sk, lk, np.float32(w.sparsity))


def _oracle(w, lk, q, k, v, precision="native"):
    qb, kb, vb = (to_bnsd_np(t, w.layout) for t in (q, k, v))
    gq = oracle.geometry(w.S, w.txt_len, *w.latent)
    gk = oracle.geometry(kb.shape[2], w.txt_len, *lk)
    mask, margin = oracle.build_mask(qb, kb, gq, float(np.float32(w.sparsity)), gk)
    return qb, kb, vb, gq, gk, mask, margin


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("precision", ["native", "fp8"])
def test_mask_and_attention(rfsa, case, precision):
    w, lk, Sk, q, k, v = _inputs(case)
    pq, pk = _plans(rfsa, w, lk, Sk)
    ws = rfsa.alloc_workspace(w.B, w.S, w.N, w.D, w.txt_len, w.latent, precision=precision, S_kv=Sk, latent_k=lk)
    sp = np.float32(w.sparsity)
    rfsa.rf_prepare(q, k, v, w.layout, w.txt_len, w.latent, sp, ws, precision=precision, latent_k=lk)
    qb, kb, vb, gq, gk, mask, margin = _oracle(w, lk, q, k, v)
    dense = oracle.is_dense(gq, gk)
    if not dense:
        views = rfsa.workspace_views(ws, w.B, w.N, pq, precision=precision, plan_kv=pk)
        bad, excused, near = mask_mismatch(views["mask"].cpu().numpy().view(np.uint32), mask, margin)
        assert bad == 0, f"{bad} mask rows differ outside near-ties"
        views["mask"].copy_(torch.from_numpy(pack_mask(mask).view(np.int32)).cuda())
    out = torch.empty_like(q)
    rfsa.rf_attend(out, w.layout, w.txt_len, w.latent, sp, ws, precision=precision, S_kv=Sk, latent_k=lk)
    assert rfsa.rf_read_status(ws, w.B, w.N, 128, pq) == 0
    got = to_bnsd_np(out, w.layout).astype(np.float64)
    for n in range(w.N):
        if precision == "fp8":
            ref, bound, sigma = fp8_reference(qb[0, n], kb[0, n], vb[0, n], gq, None if dense else mask[0, n],
                                              w.D ** -0.5, gk=gk, dense=dense)
            assert_close_fp8(got[0, n], ref, bound, sigma, f"{case} fp8 n{n}")
        else:
            ref = oracle.attention_rows(qb[0, n], kb[0, n], vb[0, n], gq, None if dense else mask[0, n],
                                        w.D ** -0.5, gk=gk)
            assert_close(got[0, n], ref, f"{case} n{n}")


@pytest.mark.parametrize("case", ["longer_kv", "shorter_kv_promoted"])
def test_fp8_codes_and_scales_of_each_side(rfsa, case):
    w, lk, Sk, q, k, v = _inputs(case)
    pq, pk = _plans(rfsa, w, lk, Sk)
    ws = rfsa.alloc_workspace(w.B, w.S, w.N, w.D, w.txt_len, w.latent, precision="fp8", S_kv=Sk, latent_k=lk)
    rfsa.rf_prepare(q, k, v, w.layout, w.txt_len, w.latent, np.float32(w.sparsity), ws, precision="fp8", latent_k=lk)
    torch.cuda.synchronize()
    views = rfsa.workspace_views(ws, w.B, w.N, pq, precision="fp8", plan_kv=pk)
    qb, kb, vb, gq, gk, _, _ = _oracle(w, lk, q, k, v)
    for n in range(w.N):
        for xb, g, key, plan in ((qb, gq, "q", pq), (kb, gk, "k", pk), (vb, gk, "v", pk)):
            _, codes, sc = fp8.quantize_head(xb[0, n], g)
            np.testing.assert_array_equal(views[key + "_scales"][0, n].cpu().numpy().view(np.uint32),
                                          sc.view(np.uint32))
            got = views[key + "8"][0, n].cpu().numpy()
            if key == "v":
                np.testing.assert_array_equal(got, codes.transpose(0, 2, 1))
            else:
                np.testing.assert_array_equal(got.reshape(plan.n_tiles, 128, 128), codes)


def test_plans_follow_the_pair_rule(rfsa):
    for case in CASES:
        w, lk, Sk, q, k, v = _inputs(case)
        pq, pk = _plans(rfsa, w, lk, Sk)
        _, _, _, gq, gk, _, _ = _oracle(w, lk, q, k, v)
        assert bool(pq.dense) == bool(pk.dense) == oracle.is_dense(gq, gk), case
        if not pq.dense:
            assert (pq.nb, pk.nb, pq.ff, pk.ff) == (gq.nb, gk.nb, gq.ff, gk.ff)
            assert pk.k == oracle.kept_count(gk.nb, float(np.float32(w.sparsity)))


def test_fp16_end_to_end(rfsa):
    w, lk, Sk, q, k, v = _inputs("longer_kv", torch.float16)
    out = rfsa.rf_sparse_attention(q, k, v, w.layout, w.txt_len, w.latent, np.float32(w.sparsity), latent_k=lk)
    torch.cuda.synchronize()
    ref, _, _, _ = oracle.rf_sparse_attention(to_np(q), to_np(k), to_np(v), w.layout, w.txt_len, w.latent,
                                              float(np.float32(w.sparsity)), latent_k=lk)
    assert out.dtype == torch.float16 and out.shape == q.shape
    assert_close(to_np(out), ref, "fp16 kv geometry e2e")


def test_same_geometry_given_twice_is_the_plain_call(rfsa):
    from block_sparse_video_rf_b200 import synth
    w = synth.workload("tiny", N=2, txt_len=37, latent=(8, 21, 43), sparsity=0.7, seed=63)
    q, k, v = (t.cuda() for t in synth.make_inputs(w, device="cpu"))
    a = rfsa.rf_sparse_attention(q, k, v, w.layout, w.txt_len, w.latent, np.float32(w.sparsity))
    b = rfsa.rf_sparse_attention(q, k, v, w.layout, w.txt_len, w.latent, np.float32(w.sparsity), latent_k=w.latent)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
