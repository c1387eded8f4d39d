"""The measurement hook rf_debug_set_stage_event: rf_prepare records the
caller's event between K1 and the kernels after it, so CUDA events split the
prepare call into K1 and the rest; cleared, it records nothing."""

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


@pytest.mark.parametrize("precision", ["native", "fp8"])
def test_event_splits_prepare(rfsa, precision):
    from block_sparse_video_rf_b200 import synth
    w = synth.workload("minimax", N=4, seed=71)
    q, k, v = (t.cuda() for t in synth.make_inputs(w, device="cpu"))
    sp = np.float32(w.sparsity)
    ws = rfsa.alloc_workspace(w.B, w.S, w.N, w.D, w.txt_len, w.latent, device=q.device, precision=precision)
    stream = torch.cuda.current_stream()
    e0, mid, e1 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    mid.record(stream)                                   # creates the CUDA event
    torch.cuda.synchronize()
    rfsa.rf_debug_set_stage_event(mid)
    try:
        e0.record(stream)
        rfsa.rf_prepare(q, k, v, w.layout, w.txt_len, w.latent, sp, ws, precision=precision)
        e1.record(stream)
        torch.cuda.synchronize()
    finally:
        rfsa.rf_debug_set_stage_event(None)
    k1, rest, whole = e0.elapsed_time(mid), mid.elapsed_time(e1), e0.elapsed_time(e1)
    assert k1 > 0 and rest > 0
    assert abs(k1 + rest - whole) < 1e-3 * whole + 1e-3
    # cleared: a later prepare leaves the event where it was
    before = e0.elapsed_time(mid)
    rfsa.rf_prepare(q, k, v, w.layout, w.txt_len, w.latent, sp, ws, precision=precision)
    torch.cuda.synchronize()
    assert e0.elapsed_time(mid) == before
