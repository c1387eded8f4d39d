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
    declared = set(re.findall(r"^\S[^\n(]*?\b(rf_[a-z_]+)\s*\(", hdr, flags=re.M))
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


def test_workspace_layout_is_aligned_and_sized(rfsa):
    p = rfsa.rf_plan(62752, 256, (62, 24, 42), 0.8)
    lay = rfsa.rf_workspace_layout(1, 56, 128, p)
    offs = [getattr(lay, f) for f in rfsa.WS_FIELDS]
    assert all(o % 256 == 0 for o in offs)
    assert offs == sorted(offs)
    tensor = 56 * 62848 * 128 * 2
    assert lay.k_int - lay.q_int >= tensor and lay.total > 3 * tensor
    assert rfsa.rf_workspace_size(1, 62752, 56, 128, 256, (62, 24, 42)) == lay.total


def test_ex_entry_points_validate_dtype_and_precision(rfsa):
    L = rfsa.LIB
    P = ctypes.c_void_p
    fake = P(0x1000)
    geo = (0, 1, 4096, 2, 128, 0, 4, 32, 32, 128, 0.5, 0.0)
    # dtype 5 / precision 3 -> RF_ERR_ARG before any CUDA call
    assert L.rf_sparse_attention_ex(fake, fake, fake, 5, 0, *geo, P(0x2000), None, 0, None) == 2
    assert b"dtype" in L.rf_last_error_string()
    assert L.rf_sparse_attention_ex(fake, fake, fake, 0, 3, *geo, P(0x2000), None, 0, None) == 2
    assert b"precision" in L.rf_last_error_string()
    assert L.rf_prepare_ex(fake, fake, fake, 1, 1, *geo[:-1], P(0x10000), 16, None) == 5   # fp8 workspace too small
    assert L.rf_attend_ex(1, 9, *geo, P(0x2000), P(0x10000), 1 << 40, None) == 2
    assert rfsa.rf_workspace_size(1, 4096, 2, 128, 0, (4, 32, 32), precision="fp8") > 0
    with pytest.raises(rfsa.RfError):
        rfsa.rf_workspace_layout(1, 2, 128, rfsa.rf_plan(4096, 0, (4, 32, 32), 0.5), precision="fp4")


def test_fp8_workspace_layout(rfsa):
    p = rfsa.rf_plan(62752, 256, (62, 24, 42), 0.8)
    nat = rfsa.rf_workspace_layout(1, 56, 128, p)
    lay = rfsa.rf_workspace_layout(1, 56, 128, p, precision="fp8")
    offs = [getattr(lay, f) for f in rfsa.WS_FIELDS]
    assert all(o % 256 == 0 for o in offs) and offs == sorted(offs)
    codes = 56 * 62848 * 128
    assert lay.k8 - lay.q8 >= codes and lay.v8 - lay.k8 >= codes and lay.scales - lay.v8 >= codes
    assert lay.vmax - lay.scales >= 3 * 56 * p.n_tiles * 4 and lay.total - lay.vmax >= 56 * 4
    # the native layout is the same up to the fp8 regions, which it leaves empty
    assert [getattr(nat, f) for f in rfsa.WS_FIELDS[:10]] == offs[:10]
    assert nat.q8 == nat.k8 == nat.v8 == nat.scales == nat.vmax == nat.total
    assert rfsa.rf_workspace_size(1, 62752, 56, 128, 256, (62, 24, 42), precision="fp8") == lay.total


def test_block_count_limit(rfsa):
    # 4096 sparse blocks are accepted, more are not (RF_ERR_UNSUPPORTED)
    p = rfsa.rf_plan(64 * 64 * 128, 0, (128, 64, 64), 0.5)
    assert p.nb == 4096
    with pytest.raises(rfsa.RfError) as e:
        rfsa.rf_plan(64 * 64 * 129, 0, (129, 64, 64), 0.5)     # 4128 blocks
    assert e.value.code == 3
