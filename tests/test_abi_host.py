"""Host-side checks of the C ABI: the library loads, exports every symbol the
header declares, validates arguments before touching the GPU, and plans the
same geometry as the oracle.  No compute call is made, so these run without
a GPU."""

import ctypes
import os
import re

import numpy as np
import pytest

from block_sparse_video_rf_b200 import build as rf_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def rfsa():
    rf_build.build()
    from block_sparse_video_rf_b200 import rfsa as mod
    return mod


def test_exports_match_header(rfsa):
    hdr = open(os.path.join(ROOT, "include", "rfsa.h")).read()
    declared = set(re.findall(r"^\S[^\n(]*?\b(rf_[a-z0-9_]+)\s*\(", hdr, flags=re.M))
    assert declared == set(rfsa.EXPORTS)
    lib = ctypes.CDLL(rfsa.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name


@pytest.mark.parametrize("txt,T,H,W", [(256, 62, 24, 42), (0, 4, 32, 32), (512, 8, 48, 64), (0, 21, 45, 80),
                                       (37, 3, 21, 43), (5, 5, 24, 40), (0, 1, 64, 64), (7, 3, 16, 16)])
@pytest.mark.parametrize("sparsity", [0.0, 0.5, 0.8, 0.9, 1.0])
def test_plan_matches_oracle(rfsa, txt, T, H, W, sparsity):
    import oracle
    S = txt + T * H * W
    p = rfsa.rf_plan(S, txt, (T, H, W), np.float32(sparsity))
    g = oracle.geometry(S, txt, T, H, W)
    assert bool(p.dense) == g.dense
    if g.dense:
        assert p.P == S and p.nb == 0
        return
    assert p.nb == g.nb and p.ff == g.ff
    assert p.P == len(g.prefix)
    assert p.n_promoted == len(g.promoted) and p.n_tail == len(g.tail)
    assert p.k == oracle.kept_count(g.nb, float(np.float32(sparsity)))
    assert p.P_pad % 128 == 0 and p.S_int == p.P_pad + 128 * p.nb


def test_plan_worked_numbers(rfsa, golden):
    ex = golden["minimax_h3_1344x768"]
    T, H, W = ex["latent"]
    p = rfsa.rf_plan(256 + T * H * W, 256, (T, H, W), 0.8)
    assert p.nb == ex["sparse_blocks"] and p.n_promoted + p.n_tail == ex["promoted_rows"]
    assert p.nb * 128 == ex["sparse_rows"]
    assert p.ff == 8 and p.k == 93 and p.P == 256 + 2976 and p.P_pad == 3328 and p.S_int == 62848


@pytest.mark.parametrize("bad", [-0.1, 1.1, float("nan"), float("inf")])
def test_plan_rejects_bad_sparsity(rfsa, bad):
    with pytest.raises(rfsa.RfError) as e:
        rfsa.rf_plan(4096, 0, (4, 32, 32), bad)
    assert e.value.code == 2


def test_plan_rejects_bad_geometry(rfsa):
    with pytest.raises(rfsa.RfError) as e:
        rfsa.rf_plan(4097, 0, (4, 32, 32), 0.5)
    assert e.value.code == 2
    with pytest.raises(rfsa.RfError) as e:
        rfsa.rf_plan(4096, 0, (4, 32, 32), 0.5, block_size=64)
    assert e.value.code == 3
    with pytest.raises(rfsa.RfError) as e:
        rfsa.rf_plan(100, 101, (0, 0, 0), 0.5)
    assert e.value.code == 2


def test_no_geometry_is_dense(rfsa):
    p = rfsa.rf_plan(1000, 10, (0, 0, 0), 0.8)
    assert p.dense == 1 and p.P == 1000 and p.P_pad == 1024 and p.n_tiles == 8


def test_entry_points_validate_before_any_cuda_call(rfsa):
    L = rfsa.LIB
    P = ctypes.c_void_p
    fake = P(0x1000)
    # bad layout -> RF_ERR_LAYOUT
    assert L.rf_sparse_attention(fake, fake, fake, 7, 1, 4096, 2, 128, 0, 4, 32, 32, 128, 0.5, 0.0, P(0x2000),
                                 None) == 1
    assert b"layout" in L.rf_last_error_string()
    # head dim != 128 -> RF_ERR_UNSUPPORTED
    assert L.rf_sparse_attention(fake, fake, fake, 0, 1, 4096, 2, 64, 0, 4, 32, 32, 128, 0.5, 0.0, P(0x2000),
                                 None) == 3
    # sparsity out of range -> RF_ERR_ARG
    assert L.rf_sparse_attention(fake, fake, fake, 0, 1, 4096, 2, 128, 0, 4, 32, 32, 128, 1.5, 0.0, P(0x2000),
                                 None) == 2
    # S mismatch -> RF_ERR_ARG
    assert L.rf_sparse_attention(fake, fake, fake, 0, 1, 4000, 2, 128, 0, 4, 32, 32, 128, 0.5, 0.0, P(0x2000),
                                 None) == 2
    # NULL input -> RF_ERR_ARG
    assert L.rf_sparse_attention(None, fake, fake, 0, 1, 4096, 2, 128, 0, 4, 32, 32, 128, 0.5, 0.0, P(0x2000),
                                 None) == 2
    # workspace too small / misaligned -> RF_ERR_WORKSPACE
    assert L.rf_sparse_attention_ws(fake, fake, fake, 0, 1, 4096, 2, 128, 0, 4, 32, 32, 128, 0.5, 0.0, P(0x2000),
                                    P(0x10000), 16, None) == 5
    assert L.rf_sparse_attention_ws(fake, fake, fake, 0, 1, 4096, 2, 128, 0, 4, 32, 32, 128, 0.5, 0.0, P(0x2000),
                                    P(0x10001), 1 << 40, None) == 5
    # aliasing out with q -> RF_ERR_ARG
    assert L.rf_sparse_attention_ws(fake, P(0x3000), P(0x4000), 0, 1, 4096, 2, 128, 0, 4, 32, 32, 128, 0.5, 0.0,
                                    fake, P(0x10000), 1 << 40, None) == 2


def _regions_disjoint(lay, sizes):
    spans = sorted((getattr(lay, f), getattr(lay, f) + n) for f, n in sizes.items() if n)
    return all(a_end <= b_start for (_, a_end), (b_start, _) in zip(spans, spans[1:])) and spans[-1][1] <= lay.total


def test_workspace_layout_is_aligned_and_sized(rfsa):
    p = rfsa.rf_plan(62752, 256, (62, 24, 42), 0.8)
    lay = rfsa.rf_workspace_layout(1, 56, 128, p)
    offs = [getattr(lay, f) for f in rfsa.WS_FIELDS]
    assert all(o % 256 == 0 for o in offs)
    assert lay.counter == 0 and lay.status == 256          # independent of the geometry
    tensor = 56 * 62848 * 128 * 2
    rows = 56 * p.nb
    assert _regions_disjoint(lay, {"counter": 4, "status": 4, "q_int": tensor, "k_int": tensor, "v_int": tensor,
                                   "pooled_q": rows * 512, "pooled_k": rows * 512, "mask": rows * p.mask_words * 4,
                                   "kept": rows * 4, "margin": rows * 4})
    assert rfsa.rf_workspace_size(1, 62752, 56, 128, 256, (62, 24, 42)) == lay.total


def test_ex_entry_points_validate_dtype_and_precision(rfsa):
    L = rfsa.LIB
    P = ctypes.c_void_p
    fake = P(0x1000)
    geo = (0, 1, 4096, 2, 128, 0, 4, 32, 32, 0, 0, 0, 0, 128, 0.5, 0.0)
    # dtype 5 / precision 3 -> RF_ERR_ARG before any CUDA call
    assert L.rf_sparse_attention_ex(fake, fake, fake, 5, 0, *geo, P(0x2000), None, 0, None) == 2
    assert b"dtype" in L.rf_last_error_string()
    assert L.rf_sparse_attention_ex(fake, fake, fake, 0, 3, *geo, P(0x2000), None, 0, None) == 2
    assert b"precision" in L.rf_last_error_string()
    assert L.rf_prepare_ex(fake, fake, fake, 1, 1, *geo[:-1], P(0x10000), 16, None) == 5   # fp8 workspace too small
    assert L.rf_attend_ex(1, 9, *geo, P(0x2000), P(0x10000), 1 << 40, None) == 2
    # a key/value geometry whose length does not match its latent -> RF_ERR_ARG
    kv_bad = (0, 1, 4096, 2, 128, 0, 4, 32, 32, 5000, 4, 32, 40, 128, 0.5, 0.0)
    assert L.rf_sparse_attention_ex(fake, fake, fake, 0, 0, *kv_bad, P(0x2000), None, 0, None) == 2
    assert rfsa.rf_workspace_size(1, 4096, 2, 128, 0, (4, 32, 32), precision="fp8") > 0
    with pytest.raises(rfsa.RfError):
        rfsa.rf_workspace_layout(1, 2, 128, rfsa.rf_plan(4096, 0, (4, 32, 32), 0.5), precision="fp4")


def test_fp8_workspace_layout(rfsa):
    p = rfsa.rf_plan(62752, 256, (62, 24, 42), 0.8)
    nat = rfsa.rf_workspace_layout(1, 56, 128, p)
    lay = rfsa.rf_workspace_layout(1, 56, 128, p, precision="fp8")
    offs = [getattr(lay, f) for f in rfsa.WS_FIELDS]
    assert all(o % 256 == 0 for o in offs)
    codes = 56 * 62848 * 128
    rows = 56 * p.nb
    assert _regions_disjoint(lay, {"pooled_q": rows * 512, "pooled_k": rows * 512, "mask": rows * p.mask_words * 4,
                                   "kept": rows * 4, "margin": rows * 4, "q8": codes, "k8": codes, "v8": codes,
                                   "scales": 3 * 56 * p.n_tiles * 4, "vmax": 56 * 4})
    # fp8 keeps no 16-bit internal copies (zero-sized regions) and the native layout no fp8 regions; both
    # start with the work counter and the status word and end with the attention's redo list (two counters
    # and one id per query tile)
    assert lay.q_int == lay.k_int == lay.v_int == lay.pooled_q
    assert nat.q8 == nat.k8 == nat.v8 == nat.scales == nat.vmax == nat.redo
    assert (lay.counter, lay.status) == (nat.counter, nat.status)
    assert lay.total < nat.total - 2 * codes
    for L in (nat, lay):
        assert L.total - L.redo >= (2 + 56 * p.n_tiles) * 4
    assert rfsa.rf_workspace_size(1, 62752, 56, 128, 256, (62, 24, 42), precision="fp8") == lay.total


def test_block_count_limit(rfsa):
    # 4096 sparse blocks are accepted, more are not (RF_ERR_UNSUPPORTED)
    p = rfsa.rf_plan(64 * 64 * 128, 0, (128, 64, 64), 0.5)
    assert p.nb == 4096
    with pytest.raises(rfsa.RfError) as e:
        rfsa.rf_plan(64 * 64 * 129, 0, (129, 64, 64), 0.5)     # 4128 blocks
    assert e.value.code == 3


def test_key_geometry_workspace(rfsa):
    import oracle
    pq = rfsa.rf_plan(16 + 4 * 32 * 32, 16, (4, 32, 32), 0.7)
    pk = rfsa.rf_plan(16 + 5 * 32 * 40, 16, (5, 32, 40), 0.7)
    assert pq.nb == 32 and pk.nb == 50
    lay = rfsa.rf_workspace_layout(2, 3, 128, pq, "native", pk)
    heads = 6
    assert _regions_disjoint(lay, {"q_int": heads * pq.S_int * 256, "k_int": heads * pk.S_int * 256,
                                   "v_int": heads * pk.S_int * 256, "pooled_q": heads * pq.nb * 512,
                                   "pooled_k": heads * pk.nb * 512, "mask": heads * pq.nb * pk.mask_words * 4,
                                   "kept": heads * pq.nb * 4, "margin": heads * pq.nb * 4})
    n = rfsa.rf_workspace_size(2, 16 + 4096, 3, 128, 16, (4, 32, 32), "native", 16 + 6400, (5, 32, 40))
    assert n == lay.total
    # either side dense makes both dense: the query side here has 6 blocks, so a
    # sparse key geometry sizes the workspace like a key side without geometry
    assert oracle.geometry(7 + 768, 7, 3, 16, 16).dense
    n2 = rfsa.rf_workspace_size(1, 7 + 768, 1, 128, 7, (3, 16, 16), "native", 7 + 6400, (5, 32, 40))
    n3 = rfsa.rf_workspace_size(1, 7 + 768, 1, 128, 7, (3, 16, 16), "native", 7 + 6400, (0, 0, 0))
    assert n2 == n3 > 0


def test_read_stats_validates_before_any_cuda_call(rfsa):
    import ctypes
    L = rfsa.LIB
    p = rfsa.rf_plan(4096, 0, (4, 32, 32), 0.5)
    st = rfsa.RfStats()
    P = ctypes.c_void_p
    assert L.rf_read_stats(P(0x1000), 1 << 30, 1, 2, 128, ctypes.byref(p), None, None) == 2      # NULL stats
    assert L.rf_read_stats(None, 1 << 30, 1, 2, 128, ctypes.byref(p), ctypes.byref(st), None) == 5   # NULL workspace
    assert L.rf_read_stats(P(0x1000), 16, 1, 2, 128, ctypes.byref(p), ctypes.byref(st), None) == 5   # too small
    assert L.rf_read_stats(P(0x1000), 1 << 30, 1, 2, 64, ctypes.byref(p), ctypes.byref(st), None) == 3  # D != 128


def test_stage_event_hook_sets_and_clears_without_cuda(rfsa):
    # storing or clearing the hook touches no CUDA state; an event that was
    # never created is refused by the binding
    rfsa.rf_debug_set_stage_event(None)

    class NoEvent:
        cuda_event = 0

    with pytest.raises(ValueError):
        rfsa.rf_debug_set_stage_event(NoEvent())
    rfsa.rf_debug_set_stage_event(None)


@pytest.mark.parametrize("B,S,N", [(0, 4096, 2), (1, 4096, 0), (1, 0, 2), (-1, 4096, 2), (1, -5, 2)])
def test_empty_or_negative_sizes_are_argument_errors(rfsa, B, S, N):
    # nothing to compute is refused up front, before any CUDA call
    L = rfsa.LIB
    P = ctypes.c_void_p
    fake = P(0x1000)
    st = L.rf_sparse_attention(fake, fake, fake, 0, B, S, N, 128, 0, 4, 32, 32, 128, 0.5, 0.0, P(0x2000), None)
    assert st == 2, st
    assert L.rf_last_error_string()


def test_misaligned_tensors_are_argument_errors_before_any_cuda_call(rfsa):
    # the kernels move 16-byte vectors of each 256-byte row: a tensor that
    # does not start on a 16-byte boundary is refused up front (RF_ERR_ARG),
    # never launched on
    L = rfsa.LIB
    P = ctypes.c_void_p
    ok, odd = P(0x1000), P(0x1008)
    geo = (0, 1, 4096, 2, 128, 0, 4, 32, 32, 128, 0.5, 0.0)
    for args in ((odd, ok, ok, P(0x2000)), (ok, odd, ok, P(0x2000)), (ok, ok, odd, P(0x2000)), (ok, ok, ok, odd)):
        assert L.rf_sparse_attention(*args[:3], *geo, args[3], None) == 2
        assert b"16-byte" in L.rf_last_error_string()
    assert L.rf_prepare(ok, odd, ok, *geo[:-1], P(0x10000), 1 << 40, None) == 2
    assert L.rf_attend(*geo, odd, P(0x10000), 1 << 40, None) == 2
    assert L.rf_unpermute(odd, 0, 1, 4096, 2, 128, 0, 4, 32, 32, P(0x2000), None) == 2
    assert L.rf_block_mask_noalloc(odd, ok, *geo[:-1], ok, ok, ok, None) == 2
    assert L.rf_block_mask_noalloc(ok, ok, *geo[:-1], P(0x3002), ok, ok, None) == 2     # mask not 4-byte aligned
    ex = (0, 0, 0, 1, 4096, 2, 128, 0, 4, 32, 32, 0, 0, 0, 0, 128, 0.5, 0.0)
    assert L.rf_sparse_attention_ex(ok, ok, ok, *ex, odd, None, 0, None) == 2


def test_debug_exp2_validates_before_any_cuda_call(rfsa):
    L = rfsa.LIB
    P = ctypes.c_void_p
    assert L.rf_debug_exp2_poly(P(0x1000), P(0x2000), -1, None) == 2
    assert L.rf_debug_exp2_poly(None, P(0x2000), 4, None) == 2
    assert L.rf_debug_exp2_poly(P(0x1002), P(0x2000), 4, None) == 2


def test_read_stats_ex_validates_before_any_cuda_call(rfsa):
    L = rfsa.LIB
    P = ctypes.c_void_p
    p = rfsa.rf_plan(4096, 0, (4, 32, 32), 0.5)
    st = rfsa.RfStats()
    assert L.rf_read_stats_ex(5, P(0x1000), 1 << 30, 1, 2, 128, ctypes.byref(p), None, ctypes.byref(st), None) == 2
    assert L.rf_read_stats_ex(1, P(0x1000), 16, 1, 2, 128, ctypes.byref(p), None, ctypes.byref(st), None) == 5
    assert L.rf_read_stats_ex(1, P(0x1000), 1 << 30, 1, 2, 128, None, None, ctypes.byref(st), None) == 2
    # a buffer one byte short of the fp8 workspace is refused
    n8 = rfsa.rf_workspace_size(1, 4096, 2, 128, 0, (4, 32, 32), precision="fp8")
    assert L.rf_read_stats_ex(1, P(0x1000), n8 - 1, 1, 2, 128, ctypes.byref(p), None, ctypes.byref(st), None) == 5


def test_binding_checks_tensors_before_the_library(rfsa):
    # what bare pointers cannot tell the C ABI -- type, shape, contiguity,
    # device -- is refused by the binding before any call into the library
    import torch
    q = torch.zeros(1, 4096, 2, 128, dtype=torch.bfloat16)
    cases = [
        (q, q.clone(), q.clone().float()),                           # v of another type
        (q, q[:, :4000].clone(), q.clone()),                         # k shorter than q
        (q, q.clone(), q.clone()[:, :, :1]),                         # k and v shapes differ
        (q, q.transpose(1, 2).contiguous().transpose(1, 2), q.clone()),   # k not contiguous
        (q.float(), q.float(), q.float()),                           # fp32 is not an input type
        (q, q.clone(), q.clone()),                                   # all fine but on the CPU
    ]
    for qq, kk, vv in cases:
        with pytest.raises(rfsa.RfError) as e:
            rfsa.rf_sparse_attention(qq, kk, vv, "BSND", 0, (4, 32, 32), 0.5, out=torch.empty_like(qq))
        assert e.value.code == 2
    with pytest.raises(rfsa.RfError) as e:
        rfsa.rf_sparse_attention(q, q, q, "BSND", 0, (4, 32, 32), 0.5, out=torch.empty(1, 4096, 2, 64,
                                                                                      dtype=torch.bfloat16))
    assert e.value.code == 2 and "out" in str(e.value)
    with pytest.raises(rfsa.RfError) as e:
        rfsa.rf_sparse_attention(q, q, q, "BSND", 0, (4, 32, 32), 0.5, out=torch.empty_like(q))
    assert "CUDA" in str(e.value)


def test_plain_c_caller(rfsa, tmp_path):
    # the header compiles as C11 and a C program links the library and runs
    # its host-only entry points (tests/c/abi_host.c)
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    exe = tmp_path / "abi_host"
    lib_dir = os.path.dirname(rfsa.LIB_PATH)
    subprocess.run([gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_host.c"), "-L", lib_dir, "-lrfsa",
                    "-Wl,-rpath," + lib_dir, "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "FAIL" not in r.stdout and r.stdout.count("ok") >= 11


def test_block_fast_path_of_the_reorder_geometry(rfsa, tmp_path):
    # K1 maps a sparse block's rows to tokens from the block's two 8x8 tiles
    # (two divisions per block); a C++ program checks it against the
    # row-by-row mapping for every sparse row of 14 plans (tests/c/geometry_host.cpp)
    import shutil
    import subprocess
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("no C++ compiler")
    exe = tmp_path / "geometry_host"
    lib_dir = os.path.dirname(rfsa.LIB_PATH)
    subprocess.run([gxx, "-std=c++17", "-O1", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(lib_dir, "csrc"), os.path.join(ROOT, "tests", "c", "geometry_host.cpp"),
                    "-L", lib_dir, "-lrfsa", "-Wl,-rpath," + lib_dir, "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert int(r.stdout.split()[0]) > 500_000


def test_page_signature_checks(rfsa):
    # rfsa.sparse_attention takes lite_boost.ops.sparse_attention's parameter
    # list; the page's ValueErrors come before anything reaches the library
    import torch
    q = torch.zeros(1, 4096, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        rfsa.sparse_attention(q, q, q, head_num=2, input_layout="SBND", sparse_type="rf_v2", latent_shape_q=(4, 32, 32))
    with pytest.raises(ValueError):
        rfsa.sparse_attention(q, q, q, head_num=2, input_layout="BSND", sparse_type="rf_v3", latent_shape_q=(4, 32, 32))
    with pytest.raises(ValueError):
        rfsa.sparse_attention(q, q, q, head_num=3, input_layout="BSND", sparse_type="rf_v2", latent_shape_q=(4, 32, 32))
    with pytest.raises(ValueError):
        rfsa.sparse_attention(q, q, q, head_num=2, input_layout="BSND", sparse_type="rf_v2")
    with pytest.raises(NotImplementedError):
        rfsa.sparse_attention(q, q, q, head_num=2, input_layout="BSND", is_causal=True)
    # accepted arguments reach the tensor checks (these are CPU tensors)
    with pytest.raises(rfsa.RfError) as e:
        rfsa.sparse_attention(q, q, q, head_num=2, input_layout="BSND", sparse_type="rf_v2", latent_shape_q=(4, 32, 32),
                              sparsity=0.5, keep_sink=False, cdf_threshold=0.5)
    assert "CUDA" in str(e.value)


def test_binding_checks_buffer_sizes_and_kinds(rfsa):
    # the host-buffer call takes CPU bf16 tensors shaped like q; the
    # allocation-free mask takes output tensors of at least the mask's size:
    # both are refused in the binding, before the library sees bare pointers
    import torch
    q = torch.zeros(1, 4096, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(rfsa.RfError):
        rfsa.rf_sparse_attention_host(q, q, q.float(), "BSND", 0, (4, 32, 32), 0.5, torch.empty_like(q))
    with pytest.raises(rfsa.RfError):
        rfsa.rf_sparse_attention_host(q, q[:, :2048].contiguous(), q, "BSND", 0, (4, 32, 32), 0.5, torch.empty_like(q))
    with pytest.raises(rfsa.RfError) as e:
        # CPU q and k: refused by the tensor checks (a GPU run would reach the size checks below)
        rfsa.rf_block_mask_noalloc(q, q, "BSND", 0, (4, 32, 32), 0.5, torch.zeros(1, dtype=torch.int32),
                                   torch.zeros(1, dtype=torch.int32), torch.zeros(1))
    assert e.value.code == 2
