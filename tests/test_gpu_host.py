"""The host-buffer entry points (rf_sparse_attention_host and its _ex form
for every input type, precision and key/value geometry), which run the call
on chunks of heads with the copies of neighbouring chunks overlapping the
compute.  Heads are independent in every precision (an fp8 block scale
belongs to one head's tile, vmax to one head) and every kernel's result for
a head is the same whichever launch computes it, so the output must equal
the device call on the whole tensors bit for bit.  At the MiniMax-H3
sequence length a chunk holds 2 heads: 7 heads and B = 2 give eight chunks,
a partial one among them, and reuse both device slots."""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rfsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from block_sparse_video_rf_b200 import rfsa as mod
    return mod


@pytest.mark.parametrize("layout", ["BSND", "BNSD"])
def test_host_call_equals_device_call(rfsa, layout):
    from block_sparse_video_rf_b200 import synth
    w = synth.workload("minimax", N=7, B=2, layout=layout, seed=61)
    q, k, v = synth.make_inputs(w, device="cpu")
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    out_h = torch.empty_like(qh).pin_memory()
    rfsa.rf_sparse_attention_host(qh, kh, vh, w.layout, w.txt_len, w.latent, np.float32(w.sparsity), out_h)
    ref = rfsa.rf_sparse_attention(q.cuda(), k.cuda(), v.cuda(), w.layout, w.txt_len, w.latent,
                                   np.float32(w.sparsity))
    torch.cuda.synchronize()
    assert torch.equal(out_h.view(torch.int16), ref.cpu().view(torch.int16))


def test_host_call_with_pageable_buffers(rfsa):
    # pageable host memory: the copies no longer overlap, the result is the same
    from block_sparse_video_rf_b200 import synth
    w = synth.workload("tiny", N=3, seed=62)
    q, k, v = synth.make_inputs(w, device="cpu")
    out_h = torch.empty_like(q)
    rfsa.rf_sparse_attention_host(q, k, v, w.layout, w.txt_len, w.latent, np.float32(w.sparsity), out_h)
    ref = rfsa.rf_sparse_attention(q.cuda(), k.cuda(), v.cuda(), w.layout, w.txt_len, w.latent,
                                   np.float32(w.sparsity))
    torch.cuda.synchronize()
    assert torch.equal(out_h.view(torch.int16), ref.cpu().view(torch.int16))


@pytest.mark.parametrize("layout", ["BSND", "BNSD"])
def test_host_call_against_the_oracle(rfsa, layout):
    # the host-buffer call on its own against the CPU oracle: the mask bit for
    # bit is not visible here, so the output is compared element by element
    # (near-tie rows, where the mask may differ, excused); several heads of a
    # ragged geometry with promotion, so that every chunk and both slots run
    import oracle
    from parity_util import MAX_ABS, MEAN_ABS, NEAR_TIE
    from block_sparse_video_rf_b200 import synth
    w = synth.workload("tiny", N=5, txt_len=37, latent=(8, 21, 43), sparsity=0.7, layout=layout, seed=63)
    q, k, v = synth.make_inputs(w, device="cpu")
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    out_h = torch.empty_like(qh).pin_memory()
    sp = np.float32(w.sparsity)
    rfsa.rf_sparse_attention_host(qh, kh, vh, w.layout, w.txt_len, w.latent, sp, out_h)
    ref, mask, margin, g = oracle.rf_sparse_attention(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                                      w.layout, w.txt_len, w.latent, float(sp))
    got = oracle.to_bnsd(out_h.float().numpy(), w.layout)
    refb = oracle.to_bnsd(ref, w.layout)
    # rows of query blocks whose selection sat on a near-tie may differ in their key set
    ok_rows = np.ones((w.B, w.N, w.S), dtype=bool)
    for b in range(w.B):
        for n in range(w.N):
            for i in np.nonzero(margin[b, n] < NEAR_TIE)[0]:
                ok_rows[b, n, g.blocks[i]] = False
    err = np.abs(got - refb)[ok_rows]
    assert np.isfinite(got).all()
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())


@pytest.mark.parametrize("dtype,precision,layout", [(torch.float16, "native", "BSND"),
                                                    (torch.bfloat16, "fp8", "BSND"),
                                                    (torch.float16, "fp8", "BNSD")])
def test_host_call_ex_equals_device_call(rfsa, dtype, precision, layout):
    # 5 heads and B = 2 at the MiniMax-H3 length: chunks of 2, 2 and 1 heads per batch entry
    from block_sparse_video_rf_b200 import synth
    w = synth.workload("minimax", N=5, B=2, layout=layout, seed=64)
    q, k, v = synth.make_inputs(w, device="cpu", dtype=dtype)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    out_h = torch.empty_like(qh).pin_memory()
    sp = np.float32(w.sparsity)
    rfsa.rf_sparse_attention_host(qh, kh, vh, w.layout, w.txt_len, w.latent, sp, out_h, precision=precision)
    ref = rfsa.rf_sparse_attention(q.cuda(), k.cuda(), v.cuda(), w.layout, w.txt_len, w.latent, sp,
                                   precision=precision)
    torch.cuda.synchronize()
    assert torch.equal(out_h.view(torch.int16), ref.cpu().view(torch.int16))


@pytest.mark.parametrize("precision,layout", [("native", "BSND"), ("fp8", "BNSD")])
def test_host_call_with_own_kv_geometry_equals_device_call(rfsa, precision, layout):
    # k and v longer than q, with a geometry of their own: a chunk copies S
    # tokens of q and out and S_kv of k and v; 96 MiB holds one head of this
    # size, so BSND runs chunks of 2 heads and BNSD of 1
    from block_sparse_video_rf_b200 import synth
    lk = (20, 48, 80)
    wq = synth.workload("tiny", N=5, latent=(16, 48, 80), txt_len=16, sparsity=0.8, layout=layout, seed=65)
    wk = synth.workload("tiny", N=5, latent=lk, txt_len=16, layout=layout, seed=66)
    q, _, _ = synth.make_inputs(wq, device="cpu")
    _, k, v = synth.make_inputs(wk, device="cpu")
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    out_h = torch.empty_like(qh).pin_memory()
    sp = np.float32(wq.sparsity)
    rfsa.rf_sparse_attention_host(qh, kh, vh, layout, wq.txt_len, wq.latent, sp, out_h, precision=precision,
                                  latent_k=lk)
    ref = rfsa.rf_sparse_attention(q.cuda(), k.cuda(), v.cuda(), layout, wq.txt_len, wq.latent, sp,
                                   precision=precision, latent_k=lk)
    torch.cuda.synchronize()
    assert torch.equal(out_h.view(torch.int16), ref.cpu().view(torch.int16))
