"""The library's cached device buffers.  rf_sparse_attention (and the _ex
form with a NULL workspace) and the host-buffer calls share one workspace
cache per device, grown on first use of a larger shape and never shrunk, so
a call usually runs in a buffer that a larger or different call used
before.  Whatever a call reads must be what it wrote itself: every result of
a sequence of calls of growing and shrinking shapes, both precisions and
both layouts, must equal the same call on a fresh caller-owned workspace bit
for bit."""

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


# (workload, overrides, precision, also through the host-buffer call)
SEQUENCE = [
    ("tiny", {"seed": 80}, "native", False),
    ("tiny", {"N": 3, "txt_len": 37, "latent": (8, 21, 43), "sparsity": 0.7, "seed": 81}, "fp8", True),
    ("tiny", {"B": 2, "layout": "BNSD", "seed": 82}, "native", True),
    ("tiny", {"seed": 83}, "fp8", False),
    ("tiny", {"N": 3, "txt_len": 37, "latent": (8, 21, 43), "sparsity": 0.9, "seed": 84}, "native", False),
    ("tiny", {"N": 2, "latent": (3, 16, 16), "txt_len": 7, "sparsity": 0.9, "seed": 85}, "fp8", True),   # dense
    ("tiny", {"seed": 86}, "native", True),
]


def test_cached_buffers_across_shapes_and_precisions(rfsa):
    from block_sparse_video_rf_b200 import synth
    for name, over, precision, host in SEQUENCE:
        w = synth.workload(name, **over)
        sp = np.float32(w.sparsity)
        q, k, v = synth.make_inputs(w, device="cuda")
        got = rfsa.rf_sparse_attention(q, k, v, w.layout, w.txt_len, w.latent, sp, precision=precision)
        ws = rfsa.alloc_workspace(w.B, w.S, w.N, w.D, w.txt_len, w.latent, precision=precision)
        ref = rfsa.rf_sparse_attention_ws(q, k, v, w.layout, w.txt_len, w.latent, sp, ws, precision=precision)
        torch.cuda.synchronize()
        what = f"{name} {over} {precision}"
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), what
        if host:
            qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
            out_h = torch.empty_like(qh).pin_memory()
            rfsa.rf_sparse_attention_host(qh, kh, vh, w.layout, w.txt_len, w.latent, sp, out_h, precision=precision)
            assert torch.equal(out_h.view(torch.int16), ref.cpu().view(torch.int16)), what + " (host buffers)"
