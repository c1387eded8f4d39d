"""Failure detection on the GPU without a fault: a bounded wait in the
attention kernel is made to run out (the first query tile's copy is never
issued), the kernel records RF_ERR_TIMEOUT in the status word and returns,
and the same context then computes correct results again."""

import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_close, to_bnsd_np



@pytest.mark.gpu
@pytest.mark.parametrize("path", [0, 1], ids=["chain_kernel", "two_tile_kernel"])
def test_wait_timeout_is_reported_and_context_recovers(path):
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from block_sparse_video_rf_b200 import rfsa, synth
    rfsa.rf_debug_set_path(path, 0.0)
    w = synth.workload("tiny")
    q, k, v = (t.cuda() for t in synth.make_inputs(w, device="cpu"))
    sp = np.float32(w.sparsity)
    plan = rfsa.rf_plan(w.S, w.txt_len, w.latent, sp)
    ws = rfsa.alloc_workspace(w.B, w.S, w.N, w.D, w.txt_len, w.latent)
    out = torch.zeros_like(q)
    rfsa.rf_prepare(q, k, v, w.layout, w.txt_len, w.latent, sp, ws)
    try:
        rfsa.rf_debug_set_wait(20_000_000, 1)          # 20 ms limit, first Q copy never issued
        rfsa.rf_attend(out, w.layout, w.txt_len, w.latent, sp, ws)
        status = rfsa.rf_read_status(ws, w.B, w.N, 128, plan)
    finally:
        rfsa.rf_debug_set_wait(0, 0)
    assert status == 6                                  # RF_ERR_TIMEOUT
    # the context is still usable and the status word was cleared
    try:
        rfsa.rf_attend(out, w.layout, w.txt_len, w.latent, sp, ws)
        assert rfsa.rf_read_status(ws, w.B, w.N, 128, plan) == 0
    finally:
        rfsa.rf_debug_set_path(0, 0.0)
    ref, _, _, _ = oracle.rf_sparse_attention(q.float().cpu().numpy(), k.float().cpu().numpy(),
                                              v.float().cpu().numpy(), w.layout, w.txt_len, w.latent, float(sp))
    assert_close(out.float().cpu().numpy(), ref, "after timeout")


def test_debug_control_rejects_bad_values():
    from block_sparse_video_rf_b200 import build as rf_build
    rf_build.build()
    from block_sparse_video_rf_b200 import rfsa
    with pytest.raises(rfsa.RfError):
        rfsa.rf_debug_set_wait(-1, 0)
    with pytest.raises(rfsa.RfError):
        rfsa.rf_debug_set_wait(0, 2)
    rfsa.rf_debug_set_wait(0, 0)
    with pytest.raises(rfsa.RfError):
        rfsa.rf_debug_set_path(2, 0.0)
    with pytest.raises(rfsa.RfError):
        rfsa.rf_debug_set_path(0, -1.0)
    rfsa.rf_debug_set_path(0, 0.0)
