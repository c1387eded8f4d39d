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


def fp8_bounds(v_deq: np.ndarray):
    """Output tolerance of the fp8 path against the oracle over the
    dequantised operands, from the arithmetic the oracle leaves out: P is
    rounded to e4m3 (3 mantissa bits, round to nearest even), a relative
    error of at most 2^-4 per weight.  An output row is a weighted mean of V
    rows, so its error is at most 2^-4 * max |V| if every weight errs the
    same way; with errors of mixed sign and an average size well below
    2^-5, the mean error stays under 2^-6 * mean |V|."""
    a = np.abs(np.asarray(v_deq, dtype=np.float64))
    return 2.0 ** -4 * float(a.max()), 2.0 ** -6 * float(a.mean())


def assert_close_fp8(got, ref, v_deq, what=""):
    mx_tol, mean_tol = fp8_bounds(v_deq)
    mx, mean = compare_outputs(got, ref)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert mx <= mx_tol and mean <= mean_tol, \
        f"{what}: max-abs {mx:.3e} (<= {mx_tol:.3e}), mean-abs {mean:.3e} (<= {mean_tol:.3e})"
    return mx, mean


def mask_mismatch(gpu_words: np.ndarray, ref_bool: np.ndarray, ref_margin: np.ndarray):
    """Rows whose mask differs, split into excused near-ties and real mismatches."""
    nb = ref_bool.shape[-1]
    got = unpack_mask(gpu_words, nb)
    diff_rows = (got != ref_bool).any(axis=-1)
    near = ref_margin < NEAR_TIE
    return int((diff_rows & ~near).sum()), int((diff_rows & near).sum()), int(near.sum())
