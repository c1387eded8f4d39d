"""fp8 e4m3 operands of the attention (the fp8 precision), written out plainly.

TEST INFRASTRUCTURE ONLY: the product path never imports this module.

Sources: [SA] MindSpore Lite "lite_boost.ops.sparse_attention" lists an fp8
precision for the attention; the pages fix no scaling rule.  READING (the
CUDA library takes the same one; the two share no code):

  R14 Q, K and V are quantised per 128-row block of the internal layout
      (the attention's tile: each prefix tile, padded with zero rows, and
      each sparse block), per tensor and (b, head):
        amax  = max |x| over the block's 128 x 128 values;
        inv   = fp32(448 / amax)           (448: the largest finite e4m3);
        code  = e4m3(fp32(x * inv))        round to nearest, ties to even,
                                           saturating at +-448;
        scale = fp32(amax / 448);
      an all-zero block has scale 0 and codes 0.  The dequantised operand is
      e4m3_value(code) * scale.  The block mask is computed from the
      unquantised inputs, exactly as at native precision.
  R15 The fp8 attention output is the oracle's attention (fp64) over the
      dequantised Q, K and V.  An fp8 tensor-core path must also round the
      softmax weights P to e4m3 before P V; the oracle does not apply that
      rounding, but ``p_rounding_model`` states what it can change: per
      output element a worst-case bound and an error scale, both computed
      from the oracle's own weights (see there for the derivation).

Parity unpinned: R14's choice of block and of rounding (a reading; the
e4m3 format itself is pinned against torch's cast).

The e4m3 format (OCP 8-bit floating point, E4M3): 1 sign bit, 4 exponent
bits with bias 7, 3 mantissa bits; exponent field 0 holds subnormals
m * 2^-9; no infinities; exponent 15 with mantissa 7 is NaN, so the largest
finite value is 1.75 * 2^8 = 448.

Parity: the value table and the rounding are pinned against torch's
float8_e4m3fn conversion and against a brute-force nearest-value search in
``tests/test_oracle_fp8.py``; the quantised attention equals the plain
oracle exactly on operands that e4m3 represents exactly; the error model of
the P rounding is checked against an explicit e4m3 rounding of P on random
rows (flat, peaked, and with the reference maximum far below the row's).
"""

from __future__ import annotations

import numpy as np

from . import rf_v2

E4M3_MAX = 448.0


def e4m3_values() -> np.ndarray:
    """The value of each of the 256 codes (fp64; NaN for the two NaN codes)."""
    vals = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            vals[code] = np.nan
        elif e == 0:
            vals[code] = sign * m * 2.0 ** -9
        else:
            vals[code] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_VALUES = e4m3_values()


def _binade(a: np.ndarray) -> np.ndarray:
    """floor(log2(a)) for a > 0, exactly (frexp: a = m 2^p with m in [0.5, 1))."""
    return np.frexp(a)[1].astype(np.int64) - 1


def e4m3_round(x) -> np.ndarray:
    """Codes (uint8) of fp32 values: round to nearest, ties to even mantissa,
    |x| above 448 saturating to 448 (R14), negative values that round to zero
    giving -0 (code 0x80).  NaN inputs are not expected."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    pos = a > 0
    e = np.where(pos, np.maximum(_binade(np.where(pos, a, 1.0)), -6), 0)   # below 2^-6: subnormal spacing 2^-9
    quantum = np.ldexp(1.0, e - 3)                                           # 3 mantissa bits
    q = np.round(a / quantum) * quantum                                      # np.round: halves to even
    q = np.where(a >= E4M3_MAX, E4M3_MAX, np.minimum(q, E4M3_MAX))
    # code of the rounded magnitude
    normal = q >= 2.0 ** -6
    eq = np.where(normal, _binade(np.where(normal, q, 1.0)), 0)
    mant = np.where(normal, q / np.ldexp(1.0, eq) * 8 - 8, q / 2.0 ** -9)
    code = np.where(normal, ((eq + 7) << 3), 0) + np.round(mant).astype(np.int64)
    code = np.where(np.signbit(x), code | 0x80, code)                      # the sign survives underflow: -0
    return code.astype(np.uint8)


def quantize_block(x: np.ndarray):
    """R14 for one block: (codes uint8 like x, scale fp32)."""
    xf = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(xf))) if xf.size else np.float32(0.0)
    if amax == 0:
        return np.zeros(xf.shape, dtype=np.uint8), np.float32(0.0)
    inv = np.float32(np.float32(E4M3_MAX) / amax)
    v = (xf * inv).astype(np.float32)
    return e4m3_round(v), np.float32(amax / np.float32(E4M3_MAX))


def dequantize(codes: np.ndarray, scale) -> np.ndarray:
    return _VALUES[np.asarray(codes, dtype=np.int64)] * float(scale)


def internal_tiles(g: rf_v2.Geometry, dense: bool | None = None) -> list[np.ndarray]:
    """Token indices of each 128-row block of the internal layout, -1 for the
    zero pad rows: the prefix in order (the whole sequence when dense),
    padded to a multiple of 128, then the sparse blocks.  ``dense``
    overrides g.dense (a call is dense when either geometry is, R10)."""
    dense = g.dense if dense is None else dense
    pre = np.arange(g.S) if dense else np.asarray(g.prefix, dtype=np.int64)
    pad = (-len(pre)) % rf_v2.BLOCK
    rows = np.concatenate([pre, -np.ones(pad, dtype=np.int64)])
    tiles = [rows[i:i + rf_v2.BLOCK] for i in range(0, len(rows), rf_v2.BLOCK)]
    if not dense:
        tiles += [np.asarray(b, dtype=np.int64) for b in g.blocks]
    return tiles


def quantize_head(xh: np.ndarray, g: rf_v2.Geometry, dense: bool | None = None):
    """R14 for one (b, head) tensor [S, D] in token order: returns the
    dequantised tensor (fp64, token order), the codes per internal tile
    ([n_tiles, 128, D], pad rows 0) and the scales [n_tiles] (fp32).
    ``dense`` as in internal_tiles."""
    S, D = xh.shape
    tiles = internal_tiles(g, dense)
    xq = np.zeros((S, D), dtype=np.float64)
    codes = np.zeros((len(tiles), rf_v2.BLOCK, D), dtype=np.uint8)
    scales = np.zeros(len(tiles), dtype=np.float32)
    for t, rows in enumerate(tiles):
        valid = rows >= 0
        block = np.zeros((rf_v2.BLOCK, D), dtype=np.float32)
        block[valid] = xh[rows[valid]]
        c, s = quantize_block(block)
        codes[t], scales[t] = c, s
        xq[rows[valid]] = dequantize(c[valid], s)
    return xq, codes, scales


def rf_sparse_attention_fp8(q, k, v, layout: str, txt_len: int, latent, sparsity: float,
                            scale: float | None = None, latent_k=None):
    """The whole call at fp8 precision (R14, R15): returns (out fp64 in the
    caller's layout, mask, margin, geometry).  ``latent_k`` as in
    ``rf_v2.rf_sparse_attention``: k and v are then quantised by the blocks
    of their own geometry."""
    if not (np.isfinite(sparsity) and 0.0 <= sparsity <= 1.0):
        raise ValueError("sparsity must be finite and in [0, 1]")
    qb, kb, vb = (rf_v2.to_bnsd(np.asarray(a), layout) for a in (q, k, v))
    B, N, S, D = qb.shape
    if scale is None:
        scale = D ** -0.5
    T, H, W = latent
    g = rf_v2.geometry(S, txt_len, T, H, W)
    gk = None if latent_k is None else rf_v2.geometry(kb.shape[2], txt_len, *latent_k)
    gkv = g if gk is None else gk
    mask, margin = rf_v2.build_mask(qb, kb, g, sparsity, gk)
    dense = rf_v2.is_dense(g, gk)
    out = np.empty((B, N, S, D), dtype=np.float64)
    for b in range(B):
        for n in range(N):
            qd = quantize_head(qb[b, n], g, dense)[0]
            kd, vd = (quantize_head(x[b, n], gkv, dense)[0] for x in (kb, vb))
            out[b, n] = rf_v2.attention_rows(qd, kd, vd, g, None if dense else mask[b, n], scale, gk=gk)
    return rf_v2.from_bnsd(out, layout), mask, margin, (g if gk is None else (g, gk))


# ---------------------------------------------------------------------------
# The rounding of P to e4m3 (R15): what it can change in the output
# ---------------------------------------------------------------------------

P_REL = 2.0 ** -4        # e4m3 normals: 3 mantissa bits, round to nearest -> |p~ - p| <= 2^-4 p
P_MIN_NORMAL = 2.0 ** -6  # below it the spacing is 2^-9 ...
P_ABS = 2.0 ** -10       # ... so |p~ - p| <= min(p, 2^-10) (values under 2^-10 round to 0)
ARITH_REL = 2.0 ** -9    # room for the fp32 scores and sums and the approximate exponentials
OUT_REL = 2.0 ** -8      # the 16-bit output's own rounding (bf16: at most 2^-9 |o|), with room


def token_scales(g: rf_v2.Geometry, scales: np.ndarray, dense: bool | None = None) -> np.ndarray:
    """[S] the block scale of each token's internal tile (``scales`` as
    returned by ``quantize_head`` for the same geometry)."""
    out = np.zeros(g.S, dtype=np.float64)
    for t, rows in enumerate(internal_tiles(g, dense)):
        valid = rows >= 0
        out[rows[valid]] = float(scales[t])
    return out


def p_rounding_model(e: np.ndarray, v: np.ndarray, sv_tok: np.ndarray, vmax: float):
    """Output rows and the error the e4m3 rounding of P may add to them.

    ``e`` [R, K]: exp(scale q.k - M) of each row over its key set, with M the
    row's largest scaled score (the oracle's own softmax numerators, fp64);
    ``v`` [K, D]: the dequantised values of those keys; ``sv_tok`` [K]: the
    block scale of each key's V tile; ``vmax``: the head's largest V block
    scale.  Returns (o, bound, sigma), each [R, D].

    Derivation.  Let w_j = e_j / L_M with L_M = sum_j e_j, so o = sum_j w_j v_j.
    An fp8 path takes a reference maximum of its choosing, m <= M (a
    maximum over part of the row is at most the row's), writes the weights
    as P'_j = 2^D e_j sv_j / vmax with D = M - m >= 0 (so that P' times V's
    own codes, v_j = sv_j code_j, carries the one factor vmax), keeps them
    at most 448 (so none saturates), rounds them to e4m3 (RNE), P~'_j =
    P'_j + d_j, and divides by the sum of the unrounded weights, L = 2^D L_M.
    The output is then o + sum_j d_j (vmax / sv_j) v_j / L, and
      * if e_j sv_j / vmax >= 2^-6, P'_j is a normal e4m3 value whatever D
        is, |d_j| <= 2^-4 P'_j, and the key's term is at most 2^-4 w_j |v_j|;
      * otherwise P'_j may lie in the subnormal range, where
        |d_j| <= min(P'_j, 2^-10) (or 2^-4 P'_j if it is normal after all);
        dividing by L = 2^D L_M, the term is at most
        max(2^-4 w_j, min(w_j, 2^-10 vmax / (sv_j L_M))) |v_j| for every D >= 0.
    With c_j those coefficients, the worst case is sum_j c_j |v_j|.  The
    approximate exponentials and the fp32 scores and sums change P'_j and
    L together by relative amounts far below 2^-9, which moves o by at most
    2^-9 sum_j w_j |v_j - o| <= 2^-9 (sum_j w_j |v_j| + |o|); the 16-bit
    output adds at most 2^-9 |o| (bf16), taken as 2^-8 |o|.
    The rounding errors of different keys are independent and (up to the
    truncation of the smallest values to 0) of zero mean; the term of key j
    lies in [-c_j |v_j|, c_j |v_j|], whose uniform distribution has variance
    (c_j v_j)^2 / 3, and RNE's error is no wider.  The error of an element
    therefore has a standard deviation of at most
    sigma = sqrt(sum_j (c_j v_j)^2 / 3 + (2^-9 o)^2 / 3), the second term
    for the output's rounding.
    """
    e = np.asarray(e, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    sv = np.asarray(sv_tok, dtype=np.float64)
    L = e.sum(axis=1, keepdims=True)
    w = e / L
    o = w @ v
    av = np.abs(v)
    c = P_REL * w
    if vmax > 0:
        ratio = np.where(sv > 0, sv / vmax, 0.0)                  # sv_j / vmax in [0, 1]
        sub = e * ratio[None, :] < P_MIN_NORMAL                    # may be subnormal for some reference
        with np.errstate(divide="ignore"):
            cap = np.where(ratio > 0, P_ABS / np.where(ratio > 0, ratio, 1.0), np.inf)[None, :] / L
        c = np.where(sub, np.maximum(c, np.minimum(w, cap)), c)
    wav = w @ av
    bound = (c @ av) * (1.0 + 2.0 ** -6) + ARITH_REL * (wav + np.abs(o)) + OUT_REL * np.abs(o) + 2.0 ** -24
    sigma = np.sqrt(((c * c) @ (v * v)) / 3.0 + (2.0 ** -9 * o) ** 2 / 3.0 + (2.0 ** -24) ** 2)
    return o, bound, sigma


def attention_rows_fp8(qd, kd, vd, sv_tok, vmax: float, g: rf_v2.Geometry, mask_bn, scale: float, rows=None,
                       chunk: int = 128, gk: rf_v2.Geometry | None = None):
    """R15 for one (b, head): the attention of ``rows`` (default all) over
    the dequantised operands, as ``rf_v2.attention_rows`` computes it, with
    the per-element bound and error scale of ``p_rounding_model``.

    ``sv_tok`` [S_kv]: the V block scale of each key token (``token_scales``);
    ``vmax``: the head's largest V block scale.  Returns (o, bound, sigma),
    each [len(rows), D] in fp64.
    """
    q64, k64, v64 = (np.asarray(a, dtype=np.float64) for a in (qd, kd, vd))
    S, D = q64.shape
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.empty((len(rows), D))
    bound = np.empty((len(rows), D))
    sigma = np.empty((len(rows), D))
    dense = rf_v2.is_dense(g, gk)
    block_of = np.full(S, -1, dtype=np.int64)
    if not dense:
        block_of[g.blocks.ravel()] = np.repeat(np.arange(g.nb), rf_v2.BLOCK)
    groups: dict[int, list[int]] = {}
    for pos, r in enumerate(rows):
        groups.setdefault(int(block_of[r]), []).append(pos)
    for blk, positions in groups.items():
        keys = rf_v2.key_set(g, mask_bn, None if blk < 0 else blk, gk)
        kk, vv, sv = k64[keys], v64[keys], np.asarray(sv_tok, dtype=np.float64)[keys]
        positions = np.asarray(positions)
        for c0 in range(0, len(positions), chunk):
            p = positions[c0:c0 + chunk]
            s = (q64[rows[p]] @ kk.T) * scale
            e = np.exp(s - s.max(axis=1, keepdims=True))
            out[p], bound[p], sigma[p] = p_rounding_model(e, vv, sv, vmax)
    return out, bound, sigma
