"""Sequence-parallel use of the rf_v2 call (Ulysses all-to-all).

vllm-omni "RainFusion Attention", "Requirements and compatibility": the
attention works under Ulysses sequence parallelism and not under ring
attention, because the block ranking needs every key of a head.  Ulysses
gives each rank every key of a subset of the heads: one all-to-all turns the
caller's sequence shards into head shards, the library's call runs on whole
sequences of the local heads (the heads are independent: each has its own
mask), and a second all-to-all turns the result back into sequence shards.

Layout: with P ranks, rank r holds tokens [r S/P, (r + 1) S/P) of every head,
BSND ``[B, S/P, N, D]``; between the two exchanges it holds all S tokens of
heads [r N/P, (r + 1) N/P).  S and N must be multiples of P.

The exchanges are torch.distributed collectives (NCCL over NVLink on GPUs;
gloo on CPU in the tests): this module moves tensors only, the computation
is the library's.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def seq_to_heads(x: torch.Tensor, group=None) -> torch.Tensor:
    """[B, S/P, N, D] sequence shard -> [B, S, N/P, D] head shard."""
    P = dist.get_world_size(group)
    B, Sl, N, D = x.shape
    if N % P:
        raise ValueError(f"head count {N} is not a multiple of the {P} ranks")
    send = x.reshape(B, Sl, P, N // P, D).permute(2, 0, 1, 3, 4).contiguous()   # chunk p: head group p
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)                           # chunk j: rank j's tokens
    return recv.permute(1, 0, 2, 3, 4).reshape(B, P * Sl, N // P, D)


def heads_to_seq(y: torch.Tensor, group=None) -> torch.Tensor:
    """[B, S, N/P, D] head shard -> [B, S/P, N, D] sequence shard."""
    P = dist.get_world_size(group)
    B, S, Nl, D = y.shape
    if S % P:
        raise ValueError(f"sequence length {S} is not a multiple of the {P} ranks")
    Sl = S // P
    send = y.reshape(B, P, Sl, Nl, D).permute(1, 0, 2, 3, 4).contiguous()     # chunk p: tokens of rank p
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)                           # chunk j: head group j
    return recv.permute(1, 2, 0, 3, 4).reshape(B, Sl, P * Nl, D)


def rf_sparse_attention_ulysses(q, k, v, txt_len: int, latent, sparsity: float, group=None, scale=None,
                                precision: str = "native", attend=None, marks=None):
    """The rf_v2 call on sequence-sharded BSND q, k, v (see the module
    docstring); returns this rank's sequence shard of the output.

    ``attend`` is the call on whole-sequence head shards; it defaults to the
    library's ``rf_sparse_attention`` (tests pass a CPU stand-in to check the
    exchanges without a GPU).  ``marks``, if given, is called with 0 before
    the first exchange, 1 after it, 2 after the call and 3 after the second
    exchange (a benchmark records CUDA events there)."""
    if attend is None:
        from . import rfsa

        def attend(qh, kh, vh):
            return rfsa.rf_sparse_attention(qh, kh, vh, "BSND", txt_len, latent, sparsity, scale=scale,
                                            precision=precision)

    mark = marks if marks is not None else (lambda i: None)
    mark(0)
    qh, kh, vh = (seq_to_heads(t.contiguous(), group) for t in (q, k, v))
    mark(1)
    oh = attend(qh, kh, vh)
    mark(2)
    o = heads_to_seq(oh, group)
    mark(3)
    return o
