"""Shared helpers of the parity tests: run the oracle on the same seeded bf16
inputs the CUDA path gets, and compare."""

from __future__ import annotations

import numpy as np
import torch

import oracle

# Output tolerance against the fp32/fp64 oracle for bf16 inputs and output.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
NEAR_TIE = 1e-5


def to_np(x: torch.Tensor) -> np.ndarray:
    return x.detach().float().cpu().numpy()


def pack_mask(mask_bool: np.ndarray) -> np.ndarray:
    """[..., nb] bool -> [..., ceil(nb/32)] uint32, bit j of word j // 32."""
    nb = mask_bool.shape[-1]
    words = (nb + 31) // 32
    out = np.zeros(mask_bool.shape[:-1] + (words,), dtype=np.uint64)
    for j in range(nb):
        out[..., j // 32] |= mask_bool[..., j].astype(np.uint64) << np.uint64(j % 32)
    return out.astype(np.uint32)


def unpack_mask(words: np.ndarray, nb: int) -> np.ndarray:
    w = words.astype(np.uint32)
    j = np.arange(nb)
    return ((w[..., j // 32] >> (j % 32).astype(np.uint32)) & 1).astype(bool)


def internal_order(g) -> np.ndarray:
    """Expected internal row -> token map (-1 = pad row) of the CUDA layout:
    prefix (text, promoted, tail) padded to 128, then the sparse blocks."""
    if g.dense:
        pre = np.arange(g.S)
        blocks = np.zeros(0, np.int64)
    else:
        pre = g.prefix
        blocks = g.blocks.ravel()
    pad = (-len(pre)) % 128
    return np.concatenate([pre, -np.ones(pad, np.int64), blocks])


def to_bnsd_np(x: torch.Tensor, layout: str) -> np.ndarray:
    return oracle.to_bnsd(to_np(x), layout)


def compare_outputs(got: np.ndarray, ref: np.ndarray):
    err = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    return float(err.max()), float(err.mean())


def assert_close(got, ref, what=""):
    mx, mean = compare_outputs(got, ref)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max-abs {mx:.3e} (<= {MAX_ABS}), mean-abs {mean:.3e} (<= {MEAN_ABS})"
    return mx, mean


# The fp8 error model's statistical check: the mean of (error / sigma)^2 over
# the compared elements.  sigma bounds each element's standard deviation
# (oracle.fp8.p_rounding_model), so the mean stays below 1 when only the
# rounding of P to e4m3 separates the kernel from the oracle; a wrong block
# scale or a missing key tile drives it far above.
FP8_SIGMA_RATIO = 1.0


def fp8_reference(qh, kh, vh, g, mask_bn, scale, rows=None, gk=None, dense=None):
    """The oracle's fp8 attention of one (b, head) (reading R15): Q, K and V
    quantised by their geometries' internal blocks, then attention over the
    dequantised values, with the per-element bound and error scale of the
    e4m3 rounding of P.  Returns (ref, bound, sigma) for ``rows`` (all when
    None), [len(rows), D] each."""
    from oracle import fp8
    gkv = g if gk is None else gk
    if dense is None:
        dense = oracle.is_dense(g, gk)
    qd = fp8.quantize_head(np.asarray(qh, np.float32), g, dense)[0]
    kd = fp8.quantize_head(np.asarray(kh, np.float32), gkv, dense)[0]
    vd, _, vsc = fp8.quantize_head(np.asarray(vh, np.float32), gkv, dense)
    sv_tok = fp8.token_scales(gkv, vsc, dense)
    return fp8.attention_rows_fp8(qd, kd, vd, sv_tok, float(vsc.max()), g, None if dense else mask_bn, scale,
                                  rows=rows, gk=gk)


def assert_close_fp8(got, ref, bound, sigma, what=""):
    """fp8 parity: every element within its worst-case bound, and the mean of
    (error / sigma)^2 at most FP8_SIGMA_RATIO.  Returns (max-abs, mean-abs,
    that mean)."""
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    worst = float((err / bound).max())
    ratio = float(np.mean((err / sigma) ** 2))
    assert worst <= 1.0, f"{what}: an element exceeds its bound by {worst:.3f}x"
    assert ratio <= FP8_SIGMA_RATIO, f"{what}: mean (err / sigma)^2 = {ratio:.3f} (<= {FP8_SIGMA_RATIO})"
    return float(err.max()), float(err.mean()), ratio


def mask_mismatch(gpu_words: np.ndarray, ref_bool: np.ndarray, ref_margin: np.ndarray):
    """Rows whose mask differs, split into excused near-ties and real mismatches."""
    nb = ref_bool.shape[-1]
    got = unpack_mask(gpu_words, nb)
    diff_rows = (got != ref_bool).any(axis=-1)
    near = ref_margin < NEAR_TIE
    return int((diff_rows & ~near).sum()), int((diff_rows & near).sum()), int(near.sum())
