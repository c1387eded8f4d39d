"""The host-buffer entry point (rf_sparse_attention_host), which runs the
call on chunks of heads with the copies of neighbouring chunks overlapping
the compute.  Heads are independent and every kernel's result for a head is
the same whichever launch computes it, so the output must equal the device
call on the whole tensors bit for bit.  At the MiniMax-H3 sequence length a
chunk holds 2 heads: 7 heads and B = 2 give eight chunks, a partial one
among them, and reuse both device slots."""

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
