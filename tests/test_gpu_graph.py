"""CUDA graph capture of the call.  With a caller-owned workspace the device
entry points only enqueue kernels and memsets on the caller's stream: the
plan and the TMA descriptors are built on the host at call time, and the
attention's second pass reads its work list on the device.  So the whole
call can be captured once and replayed.  A replay must equal an eager call
bit for bit, and must follow inputs rewritten in place (the graph holds the
addresses, not the values)."""

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


@pytest.mark.parametrize("precision,layout", [("native", "BSND"), ("fp8", "BNSD")])
def test_graph_replay_equals_eager_call(rfsa, precision, layout):
    from block_sparse_video_rf_b200 import synth
    w = synth.workload("tiny", N=3, txt_len=37, latent=(8, 21, 43), sparsity=0.7, layout=layout, seed=71)
    sp = np.float32(w.sparsity)
    q, k, v = synth.make_inputs(w, device="cuda")
    ws_eager = rfsa.alloc_workspace(w.B, w.S, w.N, w.D, w.txt_len, w.latent, precision=precision)
    ws_graph = rfsa.alloc_workspace(w.B, w.S, w.N, w.D, w.txt_len, w.latent, precision=precision)

    def eager(q_, k_, v_):
        return rfsa.rf_sparse_attention_ws(q_, k_, v_, w.layout, w.txt_len, w.latent, sp, ws_eager,
                                           precision=precision)

    first = eager(q, k, v)
    out = torch.empty_like(q)
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            rfsa.rf_sparse_attention_ws(q, k, v, w.layout, w.txt_len, w.latent, sp, ws_graph, out=out,
                                        precision=precision)
    torch.cuda.current_stream().wait_stream(side)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), first.view(torch.int16))

    # other values at the same addresses: the replay follows them
    q2, k2, v2 = synth.make_inputs(synth.workload("tiny", N=3, txt_len=37, latent=(8, 21, 43), sparsity=0.7,
                                                  layout=layout, seed=72), device="cuda")
    second = eager(q2, k2, v2).clone()
    for dst, src in ((q, q2), (k, k2), (v, v2)):
        dst.copy_(src)
    graph.replay()
    torch.cuda.synchronize()
    assert not torch.equal(second, first)
    assert torch.equal(out.view(torch.int16), second.view(torch.int16))
    plan = rfsa.rf_plan(w.S, w.txt_len, w.latent, sp)
    assert rfsa.rf_read_status(ws_graph, w.B, w.N, 128, plan) == 0
    del graph
