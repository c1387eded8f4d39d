"""The allocation-free block mask entry point, rf_block_mask_noalloc.

It exists for callers that cannot allocate device memory themselves: for
example a plugin whose process gives all device memory to one allocator that
forbids side allocations, or a loop that cannot pay for cudaMalloc's implicit
synchronisation.  Its scratch is a static device array inside the library, so
these tests check that it gives exactly the mask of the regular path
(rf_prepare, which uses a caller workspace) on consecutive calls whose inputs
and shapes differ.  A call does not depend on what the previous call left in
the shared array.  This file is named to be collected last.
"""

import numpy as np
import pytest
import torch

CASES = [
    ("minimax", {"N": 3, "latent": (12, 24, 42)}),
    ("tiny", {"txt_len": 37, "latent": (8, 21, 43), "sparsity": 0.7, "seed": 11, "N": 2}),
    # BNSD, and two batch entries (BSND and BNSD): the kernel's own token
    # offsets for each layout and batch index
    ("tiny", {"txt_len": 19, "latent": (5, 24, 40), "sparsity": 0.6, "layout": "BNSD", "seed": 12, "N": 2}),
    ("tiny", {"B": 2, "N": 2, "txt_len": 37, "latent": (6, 24, 40), "sparsity": 0.6, "seed": 41}),
    ("tiny", {"B": 2, "N": 3, "txt_len": 5, "latent": (6, 24, 40), "sparsity": 0.5, "layout": "BNSD", "seed": 42}),
    ("minimax", {"N": 3, "latent": (12, 24, 42)}),
]


def _case(name, over):
    from block_sparse_video_rf_b200 import synth
    w = synth.workload(name, **over)
    q, k, v = synth.make_inputs(w, device="cuda")
    return w, q, k, v


@pytest.mark.gpu
def test_noalloc_mask_matches_workspace_path_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from block_sparse_video_rf_b200 import rfsa
    for name, over in CASES:
        w, q, k, v = _case(name, over)
        sp = np.float32(w.sparsity)
        plan = rfsa.rf_plan(w.S, w.txt_len, w.latent, sp)
        assert plan.nb > 0
        ws = rfsa.alloc_workspace(w.B, w.S, w.N, w.D, w.txt_len, w.latent)
        rfsa.rf_prepare(q, k, v, w.layout, w.txt_len, w.latent, sp, ws)
        ref = rfsa.workspace_views(ws, w.B, w.N, plan)
        mask = torch.full_like(ref["mask"], -1)
        kept = torch.full_like(ref["kept"], -1)
        margin = torch.full_like(ref["margin"], float("nan"))
        rfsa.rf_block_mask_noalloc(q, k, w.layout, w.txt_len, w.latent, sp, mask, kept, margin)
        torch.cuda.synchronize()
        assert torch.equal(mask, ref["mask"]), name
        assert torch.equal(kept, ref["kept"]), name
        fin = torch.isfinite(ref["margin"])
        assert torch.equal(fin, torch.isfinite(margin))
        torch.testing.assert_close(margin[fin], ref["margin"][fin], rtol=1e-6, atol=1e-7)


def test_noalloc_rejects_shapes_beyond_the_static_scratch():
    from block_sparse_video_rf_b200 import build as rf_build
    rf_build.build()
    from block_sparse_video_rf_b200 import rfsa
    import ctypes
    fake = ctypes.c_void_p(0x1000)
    # 2 x 56 heads x 465 blocks = 52,080 block rows > 32,768: refused before any launch
    rc = rfsa.LIB.rf_block_mask_noalloc(fake, fake, 0, 2, 62752, 56, 128, 256, 62, 24, 42, 128, 0.8, fake, fake,
                                        fake, None)
    assert rc == 3
    assert b"static" in rfsa.LIB.rf_last_error_string()
