"""The two kernels of the 16-bit attention and the hand-over between them.

csrc/rf_attn_chain.cu runs every query tile with one running maximum per
tile (its first key tile's row maximum, no rescaling) and lists the tiles
whose P left the type's headroom; csrc/rf_attn.cu (two query tiles per CTA,
running maximum with rescaling) then computes the listed tiles.  Each path
is compared with the oracle on its own (rf_debug_set_path), with a lowered
headroom that sends a share of the tiles through the second pass, and on
inputs whose scores really leave bf16 / fp16 headroom."""

import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_close, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rfsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from block_sparse_video_rf_b200 import rfsa as mod
    yield mod
    mod.rf_debug_set_path(0, 0.0)


def _inputs(name, **over):
    from block_sparse_video_rf_b200 import synth
    w = synth.workload(name, **over)
    q, k, v = synth.make_inputs(w, device="cpu")
    return w, q.cuda(), k.cuda(), v.cuda()


def _oracle(w, q, k, v):
    ref, _, _, _ = oracle.rf_sparse_attention(to_np(q), to_np(k), to_np(v), w.layout, w.txt_len, w.latent,
                                              float(np.float32(w.sparsity)))
    return ref


def _call_ws(rfsa, w, q, k, v):
    """One call through a caller-owned workspace; returns the output and the redo list."""
    ws = rfsa.alloc_workspace(w.B, w.S, w.N, w.D, w.txt_len, w.latent)
    out = torch.empty_like(q)
    rfsa.rf_sparse_attention_ws(q, k, v, w.layout, w.txt_len, w.latent, np.float32(w.sparsity), ws, out=out)
    torch.cuda.synchronize()
    plan = rfsa.rf_plan(w.S, w.txt_len, w.latent, np.float32(w.sparsity))
    redo = rfsa.workspace_views(ws, w.B, w.N, plan)["redo"].cpu().numpy()
    return out, redo, plan


CASES = {
    "tiny": ("tiny", {}),
    "ragged": ("tiny", {"txt_len": 37, "latent": (8, 21, 43), "sparsity": 0.7, "seed": 11}),
    "oddtiles_bnsd": ("tiny", {"txt_len": 19, "latent": (5, 24, 40), "sparsity": 0.6, "layout": "BNSD", "seed": 12}),
    "dense": ("tiny", {"sparsity": 0.0, "seed": 13}),
    "batch2": ("tiny", {"B": 2, "N": 2, "txt_len": 37, "latent": (6, 24, 40), "sparsity": 0.6, "seed": 41}),
    "short_units": ("tiny", {"txt_len": 0, "latent": (3, 16, 16), "sparsity": 0.9, "seed": 14}),
    # one first-frame block and k = 0 / 1: every sparse unit reads 1 / 2 key tiles, so sets 1 and 2 (and set
    # 2) have no tile in it and the S buffers are reused back to back
    "one_tile_units": ("tiny", {"txt_len": 0, "latent": (32, 8, 16), "sparsity": 1.0, "seed": 15}),
    "two_tile_units": ("tiny", {"txt_len": 0, "latent": (32, 8, 16), "sparsity": 0.97, "seed": 16}),
}


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("path,limit", [(0, 0.0), (1, 0.0), (0, 32.0)], ids=["chain", "two_tile", "handover"])
def test_paths_against_oracle(rfsa, case, path, limit):
    name, over = CASES[case]
    w, q, k, v = _inputs(name, **over)
    rfsa.rf_debug_set_path(path, limit)
    try:
        out = rfsa.rf_sparse_attention(q, k, v, w.layout, w.txt_len, w.latent, np.float32(w.sparsity))
        torch.cuda.synchronize()
    finally:
        rfsa.rf_debug_set_path(0, 0.0)
    assert_close(to_np(out), _oracle(w, q, k, v), f"{case} path {path} limit {limit}")


def test_redo_list(rfsa):
    w, q, k, v = _inputs("tiny", N=2, txt_len=64, latent=(6, 32, 32), sparsity=0.6, seed=21)
    out, redo, plan = _call_ws(rfsa, w, q, k, v)
    assert redo[1] == 0                        # plain inputs stay far inside bf16 headroom
    total = w.B * w.N * plan.n_tiles
    ref = _oracle(w, q, k, v)
    assert_close(to_np(out), ref, "chain only")
    # lowered headroom: every listed unit is valid and listed once, the second
    # pass takes all of them, and the result is the oracle's whatever the split
    mixed = False
    try:
        for limit in (4.0, 16.0, 24.0, 32.0, 48.0, 64.0, 256.0, 1024.0):
            rfsa.rf_debug_set_path(0, limit)
            out2, redo2, _ = _call_ws(rfsa, w, q, k, v)
            n = int(redo2[1])
            ids = redo2[2:2 + n]
            assert 0 <= n <= total
            if n:
                assert len(set(ids.tolist())) == n and ids.min() >= 0 and ids.max() < total
            assert redo2[0] >= n
            assert_close(to_np(out2), ref, f"chain + second pass, limit {limit}, {n} of {total} units")
            mixed |= 0 < n < total
    finally:
        rfsa.rf_debug_set_path(0, 0.0)
    assert mixed, "no limit split the units between the two kernels"


@pytest.mark.parametrize("dtype,gain", [(torch.bfloat16, 80.0), (torch.float16, 6.0)])
def test_scores_beyond_headroom(rfsa, dtype, gain):
    # The text prefix tile comes first and fixes each row's maximum; the video
    # keys are scaled so that later tiles' P would pass 2^64 (bf16) or 65504
    # (fp16): those tiles go to the second pass, which rescales.
    w, q, k, v = _inputs("tiny", txt_len=128, latent=(4, 32, 32), N=2, seed=31)
    q, k, v = q.to(dtype), k.to(dtype).clone(), v.to(dtype)
    k[:, w.txt_len:] *= gain
    out, redo, plan = _call_ws(rfsa, w, q, k, v)
    assert redo[1] > 0
    ref = _oracle(w, q.to(torch.float32), k.to(torch.float32), v.to(torch.float32))
    assert_close(to_np(out), ref, f"beyond headroom {dtype}")


def _fp8_check(w, q, k, v, out, what):
    from parity_util import assert_close_fp8, fp8_reference, to_bnsd_np
    qb, kb, vb = (to_bnsd_np(t, w.layout) for t in (q, k, v))
    g = oracle.geometry(w.S, w.txt_len, *w.latent)
    mask, _ = oracle.build_mask(qb, kb, g, float(np.float32(w.sparsity)))
    ob = to_bnsd_np(out, w.layout)
    for b in range(w.B):
        for n in range(w.N):
            ref, bound, sigma = fp8_reference(qb[b, n], kb[b, n], vb[b, n], g, mask[b, n], w.D ** -0.5)
            assert_close_fp8(ob[b, n], ref, bound, sigma, f"{what} b{b} n{n}")


@pytest.mark.parametrize("case", ["tiny", "ragged", "batch2", "one_tile_units"])
@pytest.mark.parametrize("path,limit", [(0, 0.0), (1, 0.0), (0, 3.0)], ids=["chain", "two_tile", "handover"])
def test_fp8_paths_against_oracle(rfsa, case, path, limit):
    # e4m3 operands: the chain kernel (fp8 form), the two-tile kernel alone, and
    # a lowered limit that hands a share of the units from one to the other
    name, over = CASES[case]
    w, q, k, v = _inputs(name, **over)
    rfsa.rf_debug_set_path(path, limit)
    try:
        out = rfsa.rf_sparse_attention(q, k, v, w.layout, w.txt_len, w.latent, np.float32(w.sparsity),
                                       precision="fp8")
        torch.cuda.synchronize()
    finally:
        rfsa.rf_debug_set_path(0, 0.0)
    _fp8_check(w, q, k, v, out, f"fp8 {case} path {path} limit {limit}")


def test_fp8_scores_beyond_headroom(rfsa):
    # later tiles' P would pass e4m3's 448 against the first tile's maximum:
    # those units go to the second pass, which rescales
    w, q, k, v = _inputs("tiny", txt_len=128, latent=(4, 32, 32), N=2, seed=31)
    k = k.clone()
    k[:, w.txt_len:] *= 6.0
    ws = rfsa.alloc_workspace(w.B, w.S, w.N, w.D, w.txt_len, w.latent, precision="fp8")
    out = torch.empty_like(q)
    rfsa.rf_sparse_attention_ws(q, k, v, w.layout, w.txt_len, w.latent, np.float32(w.sparsity), ws, out=out,
                                precision="fp8")
    torch.cuda.synchronize()
    plan = rfsa.rf_plan(w.S, w.txt_len, w.latent, np.float32(w.sparsity))
    redo = rfsa.workspace_views(ws, w.B, w.N, plan, precision="fp8")["redo"].cpu().numpy()
    assert redo[1] > 0
    _fp8_check(w, q, k, v, out, "fp8 beyond headroom")


def test_read_stats_after_a_call(rfsa):
    # rf_read_stats: the mask's kept blocks, density and near-ties as the
    # workspace holds them, and the number of tiles that took the second pass
    w, q, k, v = _inputs("tiny", N=2, txt_len=64, latent=(6, 32, 32), sparsity=0.6, seed=21)
    plan = rfsa.rf_plan(w.S, w.txt_len, w.latent, np.float32(w.sparsity))
    ws = rfsa.alloc_workspace(w.B, w.S, w.N, w.D, w.txt_len, w.latent)
    out = torch.empty_like(q)
    rfsa.rf_sparse_attention_ws(q, k, v, w.layout, w.txt_len, w.latent, np.float32(w.sparsity), ws, out=out)
    st = rfsa.rf_read_stats(ws, w.B, w.N, w.D, plan)
    views = rfsa.workspace_views(ws, w.B, w.N, plan)
    kept, margin = views["kept"].cpu(), views["margin"].cpu()
    assert st["kept_blocks"] == int(kept[..., plan.ff:].sum())
    assert st["query_blocks"] == w.B * w.N * (plan.nb - plan.ff)
    assert st["near_ties"] == int((margin[..., plan.ff:] < 1e-5).sum())
    flops = rfsa.kept_block_flops(plan, kept, w.B, w.N, w.D)
    assert abs(st["kept_pairs"] * 4 * w.D - flops) <= 1e-9 * flops
    assert abs(st["density"] - st["kept_pairs"] / (w.B * w.N * w.S * w.S)) < 1e-12
    assert 0 < st["density"] < 1 and st["redo_tiles"] == 0 and st["status"] == 0
    rfsa.rf_debug_set_path(0, 4.0)
    try:
        rfsa.rf_sparse_attention_ws(q, k, v, w.layout, w.txt_len, w.latent, np.float32(w.sparsity), ws, out=out)
        st2 = rfsa.rf_read_stats(ws, w.B, w.N, w.D, plan)
    finally:
        rfsa.rf_debug_set_path(0, 0.0)
    assert st2["redo_tiles"] == int(views["redo"][1].item()) > 0
