"""RainFusion rf_v2 block-sparse attention, written out plainly in fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.

Sources, cited by page title and section:

* [RF]  vllm-omni user guide, "RainFusion Attention" -- intro paragraphs,
  "Configuration" table, "Geometry handling".
* [SA]  MindSpore Lite, "lite_boost.ops.sparse_attention" -- the rf_v2
  pipeline line (token reorder -> block pooling -> top-k sparse mask ->
  rain_fusion_attention -> inverse reorder), the parameter list and the
  returned tensor.
* [SG]  sglang error record for ``rain_fusion_attn.py`` (metadata builder):
  the range check on sparsity.

Where the pages leave a step open, the reading taken is marked READING and
is the same one the CUDA library implements (the two share no code):

  R1 tile order: 8x8 tiles row-major inside a frame, raster order inside a
     tile, frames in time order.
  R2 an aligned-token count that is not a multiple of 128 leaves a last
     partial block; its tokens join the always-kept prefix (the "suffix").
  R3 first-frame blocks (blocks holding any token of frame 0) are both
     dense query blocks and key blocks that every query block keeps.
  R4 when frame 0 is not a whole number of blocks, every block holding one
     of its tokens counts: ceil(Ha * Wa / 128) first-frame blocks.
  R5 pooling is the mean over the block's 128 tokens; prefix rows are not
     pooled.  The score is the plain dot product of pooled vectors.
  R6 kept count k = nb - floor(sparsity * nb + 1e-6), i.e. the dropped
     count rounds down; sparsity 0 keeps every block.
  R7 equal scores are ranked by the lower block index.
  R8 sparsity 1 is accepted: k = 0 leaves the prefix and the first-frame
     blocks.
  R9 prefix rows (text, promoted, partial-block suffix) attend to every
     key; every query attends to every prefix key.
  R10 fewer than 32 sparse blocks, or no geometry, means dense attention
     over the whole sequence.
  R11 the top-k is decided on fp32 scores: pooled means summed in fp64 and
     rounded to fp32, dot products in fp64 rounded to fp32.
  R13 every (batch, head) has its own mask; the permutation is shared.
  R17 a key/value geometry of its own ([SA] ``latent_shape_k``, which
     defaults to the query's): queries are reordered, pooled and blocked by
     the query geometry, keys and values by theirs, and both share txt_len.
     Block scores are nb_q x nb_k; k counts key blocks (R6 over nb_k); the
     forced columns are the key geometry's first-frame blocks and the dense
     rows the query geometry's; every query attends to the key prefix.  If
     either side is dense (R10), the call is dense attention.

(R12, the output's rounding, is the kernel's; R14 and R15, the fp8
quantisation and the rounding of its softmax weights, are in ``fp8.py``;
R16, fp16 inputs, takes this same path.)

Parity status of each function is stated in its docstring; the pins live in
``tests/test_oracle_*.py``.  Parity unpinned: R1, R2, R4 beyond the
MiniMax-H3 count, R6 beyond sparsity 0 and 0.5 with an even block count,
R7, the key-column half of R3 and the pairing rules of R17 (its sparsity-0
and dense cases are pinned to rectangular softmax attention).  These are
readings, not facts the pages fix: the oracle states each once and the CUDA
path follows it.
"""

from __future__ import annotations

from dataclasses import dataclass
import math

import numpy as np

BLOCK = 128          # [SA] parameter ``block_size``: pooling and attention block
TILE = 8             # [RF] "Geometry handling": grids aligned to 8x8
MIN_SPARSE_BLOCKS = 32   # [RF] intro: segments below 32 blocks run dense
NEAR_TIE_REL = 1e-5      # relative gap below which a k-th/(k+1)-th pair is a near-tie


# ---------------------------------------------------------------------------
# Geometry: reorder, promote, block membership
# ---------------------------------------------------------------------------

@dataclass
class Geometry:
    S: int                 # sequence length (text + video)
    txt_len: int
    T: int
    H: int
    W: int
    dense: bool            # R10 fallback: every row attends to every key
    prefix: np.ndarray     # token indices of the always-kept prefix, in order
    blocks: np.ndarray     # [nb, 128] token indices of each sparse block
    first_frame: np.ndarray  # [nb] bool: block holds a token of frame 0
    promoted: np.ndarray   # non-aligned video tokens (natural order)
    tail: np.ndarray       # aligned tokens past the last whole block (R2)

    @property
    def nb(self) -> int:
        return int(self.blocks.shape[0])

    @property
    def ff(self) -> int:
        return int(self.first_frame.sum())


def geometry(S: int, txt_len: int, T: int, H: int, W: int) -> Geometry:
    """Token classes of one clip.

    [RF] "Geometry handling": video tokens are rearranged spatially; the
    tokens that do not fit the 8x8-aligned grid are promoted to the
    always-kept prefix instead of padding.  [RF] intro: tokens are arranged
    in (t, h, w) order and grouped into 128-token blocks.  [SA] ``txt_len``:
    text tokens sit in front and take no part in the reordering.

    Parity: pinned by the worked numbers of [RF] "Geometry handling" for the
    (62, 24, 42) grid, by bijection / tile-shape invariants and by a
    nested-loop enumeration of the tile order (R1 itself is a reading).
    """
    n_video = T * H * W
    if n_video == 0:
        # No geometry: everything is prefix and dense (R10).
        return Geometry(S, txt_len, T, H, W, True, np.arange(S), np.zeros((0, BLOCK), np.int64),
                        np.zeros(0, bool), np.zeros(0, np.int64), np.zeros(0, np.int64))
    assert S == txt_len + n_video, "sequence length must be txt_len + t*h*w"
    Ha, Wa = TILE * (H // TILE), TILE * (W // TILE)

    t, y, x = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    t, y, x = t.ravel(), y.ravel(), x.ravel()          # natural (t, h, w) order
    seq = txt_len + np.arange(n_video)                  # sequence index of each video token

    aligned = (y < Ha) & (x < Wa)
    promoted = seq[~aligned]                            # natural order (ascending index)

    a = np.nonzero(aligned)[0]
    # R1: sort aligned tokens by (t, tile row, tile column, row in tile, column in tile).
    order = np.lexsort((x[a] % TILE, y[a] % TILE, x[a] // TILE, y[a] // TILE, t[a]))
    pi = seq[a][order]
    t_pi = t[a][order]

    nb = len(pi) // BLOCK
    tail = pi[nb * BLOCK:]                              # R2
    blocks = pi[: nb * BLOCK].reshape(nb, BLOCK)
    first_frame = (t_pi[: nb * BLOCK].reshape(nb, BLOCK) == 0).any(axis=1)   # R3

    prefix = np.concatenate([np.arange(txt_len), promoted, tail]).astype(np.int64)
    dense = nb < MIN_SPARSE_BLOCKS                      # R10: the partition is kept, every row is dense
    return Geometry(S, txt_len, T, H, W, dense, prefix, blocks, first_frame, promoted, tail)


def kept_count(nb: int, sparsity: float) -> int:
    """R6: number of top-scoring key blocks each sparse query block keeps.

    [RF] "Configuration": sparsity is the nominal dropped fraction of key
    blocks, 0 disables sparsity.  [SA] ``sparsity``: 0.5 prunes half the KV
    blocks.  The dropped count rounds down (guarded against representation
    error by 1e-6), so the kept count is ceil((1 - s) * nb) in exact
    arithmetic.  Parity: pinned at s = 0 (keep all) and s = 0.5, nb even
    (keep half), which the pages fix; other roundings are a reading.
    """
    drop = math.floor(float(sparsity) * nb + 1e-6)
    return int(min(max(nb - drop, 0), nb))


# ---------------------------------------------------------------------------
# Mask: pooling, block scores, top-k
# ---------------------------------------------------------------------------

def pool_blocks(x: np.ndarray, blocks: np.ndarray) -> np.ndarray:
    """R5: mean of each block's rows.  ``x`` is [S, D] for one (b, head).

    [RF] intro: key blocks of 128 tokens are pooled; [SA] pipeline: block
    pooling.  Sum in fp64, divide by the block size, round to fp32 (the
    precision in which the selection below is taken).
    """
    xs = x[blocks].astype(np.float64)                   # [nb, 128, D]
    return (xs.sum(axis=1) / blocks.shape[1]).astype(np.float32)


def block_scores(qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """R5: s_ij = qbar_i . kbar_j, fp64 sum over fp32 inputs, rounded to fp32.

    [RF] intro: pooled key blocks are ranked per query block.  The softmax
    scale is positive and left out: it does not change the ranking.
    """
    return (qbar.astype(np.float64) @ kbar.astype(np.float64).T).astype(np.float32)


def topk_mask(scores: np.ndarray, k: int, first_frame: np.ndarray, first_frame_cols: np.ndarray | None = None):
    """Kept key blocks per query block, and the gap at the k-th score.

    [SA] pipeline: top-k sparse mask generation; [RF] intro: attend to the
    highest-scoring blocks; first-frame blocks stay dense (R3).  Row i keeps
    the first k blocks of j = 0..nb-1 ordered by (score descending, j
    ascending) (R7), plus every first-frame block; a first-frame query row
    keeps all blocks.  ``margin[i]`` = (s_(k) - s_(k+1)) / max(|s_(k)|, 1e-30)
    over the sorted row (inf when k is 0 or nb, or for first-frame rows).

    With a key geometry of its own (R17) the matrix is nb_q x nb_k:
    ``first_frame`` marks the dense rows, ``first_frame_cols`` (default:
    the same) the forced columns.

    Parity: the selection is pinned against an exhaustive subset search on
    tiny rows, including exact ties.
    """
    nbq, nb = scores.shape
    ffc = first_frame if first_frame_cols is None else first_frame_cols
    mask = np.zeros((nbq, nb), dtype=bool)
    margin = np.full(nbq, np.inf, dtype=np.float64)
    for i in range(nbq):
        if first_frame[i]:
            mask[i, :] = True
            continue
        row = scores[i]
        order = np.lexsort((np.arange(nb), -row))       # primary: score desc; then index asc
        mask[i, order[:k]] = True
        mask[i, ffc] = True
        if 0 < k < nb:
            sk, sk1 = float(row[order[k - 1]]), float(row[order[k]])
            margin[i] = (sk - sk1) / max(abs(sk), 1e-30)
    return mask, margin


def is_dense(g: Geometry, gk: Geometry | None = None) -> bool:
    """R10, R17: dense attention when either side is."""
    return g.dense or (gk is not None and gk.dense)


def build_mask(q_bnsd: np.ndarray, k_bnsd: np.ndarray, g: Geometry, sparsity: float, gk: Geometry | None = None):
    """Block mask for every (b, head): [B, N, nb_q, nb_k] bool and margins [B, N, nb_q].

    ``gk`` is the key geometry (R17); None means the query's."""
    B, N = q_bnsd.shape[:2]
    gk = g if gk is None else gk
    mask = np.ones((B, N, g.nb, gk.nb), dtype=bool)
    margin = np.full((B, N, g.nb), np.inf)
    if is_dense(g, gk):
        return mask, margin
    k = kept_count(gk.nb, sparsity)
    for b in range(B):
        for n in range(N):
            qbar = pool_blocks(q_bnsd[b, n], g.blocks)
            kbar = pool_blocks(k_bnsd[b, n], gk.blocks)
            s = block_scores(qbar, kbar)
            mask[b, n], margin[b, n] = topk_mask(s, k, g.first_frame, gk.first_frame)
    return mask, margin


# ---------------------------------------------------------------------------
# Attention over each row's key set
# ---------------------------------------------------------------------------

def key_set(g: Geometry, mask_bn: np.ndarray, row_block: int | None, gk: Geometry | None = None) -> np.ndarray:
    """Token indices (of the key sequence) a query attends to.

    ``row_block`` is the query geometry's sparse block holding the query, or
    None for a prefix (dense) query; ``gk`` the key geometry (R17, default
    the query's).  R9: prefix queries and first-frame blocks see every key;
    a sparse query block sees the key prefix plus its kept key blocks.
    """
    gk = g if gk is None else gk
    if is_dense(g, gk) or row_block is None or g.first_frame[row_block]:
        return np.arange(gk.S)
    kept = np.nonzero(mask_bn[row_block])[0]
    return np.concatenate([gk.prefix, gk.blocks[kept].ravel()])


def _softmax_attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """o = softmax(scale * q k^T) v row by row, max subtracted, in fp64."""
    s = (q @ k.T) * scale
    s -= s.max(axis=1, keepdims=True)
    e = np.exp(s)
    return (e @ v) / e.sum(axis=1, keepdims=True)


def attention_rows(qh, kh, vh, g: Geometry, mask_bn, scale: float, rows=None, chunk=512, gk: Geometry | None = None):
    """rain_fusion_attention for one (b, head): fp64 output rows.

    [SA] pipeline: rain_fusion_attention over the masked key set; [SA]
    ``scale`` (default head_dim ** -0.5).  ``qh/kh/vh`` are [S, D] in the
    caller's token order, so the inverse reorder ([SA] pipeline, last step)
    is implicit: row r of the result is token r.  ``rows`` restricts the
    output to the given token indices (all when None).  ``gk`` is the key
    geometry (R17; None: the query's); kh and vh then have its length.

    Parity: the dense case is pinned against torch's scaled-dot-product
    attention; masked cases against the same routine given an explicit
    boolean mask, and against a one-hot value probe of which blocks a row
    reads.
    """
    q64, k64, v64 = (np.asarray(a, dtype=np.float64) for a in (qh, kh, vh))
    S, D = q64.shape
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.empty((len(rows), D), dtype=np.float64)

    # which sparse block (if any) holds each token
    block_of = np.full(S, -1, dtype=np.int64)
    if not is_dense(g, gk):
        block_of[g.blocks.ravel()] = np.repeat(np.arange(g.nb), BLOCK)

    groups: dict[int, list[int]] = {}
    for pos, r in enumerate(rows):
        groups.setdefault(int(block_of[r]), []).append(pos)
    for blk, positions in groups.items():
        keys = key_set(g, mask_bn, None if blk < 0 else blk, gk)
        kk, vv = k64[keys], v64[keys]
        positions = np.asarray(positions)
        for c in range(0, len(positions), chunk):
            p = positions[c:c + chunk]
            out[p] = _softmax_attend(q64[rows[p]], kk, vv, scale)
    return out


def dense_attention(qh, kh, vh, scale: float) -> np.ndarray:
    """Plain softmax attention over every key, fp64 ([SA] dense mode)."""
    q64, k64, v64 = (np.asarray(a, dtype=np.float64) for a in (qh, kh, vh))
    out = np.empty_like(q64)
    for c in range(0, q64.shape[0], 512):
        out[c:c + 512] = _softmax_attend(q64[c:c + 512], k64, v64, scale)
    return out


# ---------------------------------------------------------------------------
# Layouts and the whole call
# ---------------------------------------------------------------------------

def to_bnsd(x: np.ndarray, layout: str) -> np.ndarray:
    """[SA] ``input_layout``: BSND [B,S,N,D] or BNSD [B,N,S,D] -> BNSD."""
    if layout == "BNSD":
        return x
    if layout == "BSND":
        return np.transpose(x, (0, 2, 1, 3))
    raise ValueError("input_layout must be BSND or BNSD")


def from_bnsd(x: np.ndarray, layout: str) -> np.ndarray:
    return to_bnsd(x, layout) if layout == "BNSD" else np.transpose(x, (0, 2, 1, 3))


def rf_sparse_attention(q, k, v, layout: str, txt_len: int, latent, sparsity: float,
                        scale: float | None = None, latent_k=None):
    """The whole rf_v2 call ([SA]): returns (out fp64 in the caller's layout, mask, margin, geometry).

    ``q, k, v`` are float arrays (bf16 values widened) in BSND or BNSD.
    [SA] ``scale`` defaults to head_dim ** -0.5; [SG] and [RF] bound
    sparsity to [0, 1].  ``latent_k`` ([SA] ``latent_shape_k``, R17) gives k
    and v a geometry of their own; the returned geometry is then the pair
    (query, key).
    """
    if not (np.isfinite(sparsity) and 0.0 <= sparsity <= 1.0):
        raise ValueError("sparsity must be finite and in [0, 1]")
    qb, kb, vb = (to_bnsd(np.asarray(a), layout) for a in (q, k, v))
    B, N, S, D = qb.shape
    if scale is None:
        scale = D ** -0.5
    T, H, W = latent
    g = geometry(S, txt_len, T, H, W)
    gk = None if latent_k is None else geometry(kb.shape[2], txt_len, *latent_k)
    mask, margin = build_mask(qb, kb, g, sparsity, gk)
    out = np.empty((B, N, S, D), dtype=np.float64)
    for b in range(B):
        for n in range(N):
            out[b, n] = attention_rows(qb[b, n], kb[b, n], vb[b, n], g, None if is_dense(g, gk) else mask[b, n],
                                       scale, gk=gk)
    return from_bnsd(out, layout), mask, margin, (g if gk is None else (g, gk))
