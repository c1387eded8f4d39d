"""Ulysses sequence parallelism (block_sparse_video_rf_b200/ulysses.py): the
two all-to-all exchanges on CPU with gloo at world size 2, and the composed
call against the single-process oracle; on a GPU, the library's call through
the same path with NCCL at world size 1."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _full_inputs():
    from block_sparse_video_rf_b200 import synth
    w = synth.workload("tiny", N=4, txt_len=64, latent=(4, 32, 32), seed=51)
    q, k, v = synth.make_inputs(w, device="cpu")
    return w, q, k, v


def _oracle_attend(w):
    import oracle

    def attend(qh, kh, vh):
        out, _, _, _ = oracle.rf_sparse_attention(qh.float().numpy(), kh.float().numpy(), vh.float().numpy(), "BSND",
                                                  w.txt_len, w.latent, float(np.float32(w.sparsity)))
        return torch.from_numpy(out)

    return attend


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from block_sparse_video_rf_b200 import ulysses
        w, q, k, v = _full_inputs()
        Sl, Nl = w.S // world, w.N // world
        mine = slice(rank * Sl, (rank + 1) * Sl)
        # sequence shard -> head shard: all tokens of this rank's heads
        qh = ulysses.seq_to_heads(q[:, mine].contiguous())
        heads_ok = torch.equal(qh, q[:, :, rank * Nl:(rank + 1) * Nl])
        # and back
        back_ok = torch.equal(ulysses.heads_to_seq(qh), q[:, mine])
        # the composed call against the oracle on the whole problem, on the
        # shards bench.py's sequence-parallel arm takes, with its stage marks
        import bench
        marks = []
        qs, ks, vs = (bench.shard_rows(t, rank, world) for t in (q, k, v))
        shard_ok = torch.equal(qs, q[:, mine])
        got = ulysses.rf_sparse_attention_ulysses(qs, ks, vs, w.txt_len, w.latent, np.float32(w.sparsity),
                                                  attend=_oracle_attend(w), marks=marks.append)
        heads_ok = heads_ok and shard_ok and marks == [0, 1, 2, 3]
        try:
            ulysses.seq_to_heads(torch.zeros(1, 4, 3, 8))       # 3 heads over 2 ranks
            reject_ok = False
        except ValueError:
            reject_ok = True
        out[rank] = (heads_ok, back_ok, reject_ok, got.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_exchanges_and_composed_call_world_2():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    w, q, k, v = _full_inputs()
    ref = _oracle_attend(w)(q, k, v).numpy()
    Sl = w.S // world
    for r in range(world):
        heads_ok, back_ok, reject_ok, got = res[r]
        assert heads_ok and back_ok and reject_ok
        np.testing.assert_allclose(got, ref[:, r * Sl:(r + 1) * Sl], rtol=0, atol=1e-12)


def test_world_one_is_the_identity():
    from block_sparse_video_rf_b200 import ulysses
    port = _free_port()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        x = torch.zeros(1, 6, 3, 8)
        assert torch.equal(ulysses.heads_to_seq(ulysses.seq_to_heads(x)), x)   # P = 1 splits anything
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
def test_library_call_through_the_exchanges_nccl():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from block_sparse_video_rf_b200 import rfsa, ulysses
    port = _free_port()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        w, q, k, v = _full_inputs()
        q, k, v = q.cuda(), k.cuda(), v.cuda()
        got = ulysses.rf_sparse_attention_ulysses(q, k, v, w.txt_len, w.latent, np.float32(w.sparsity))
        ref = rfsa.rf_sparse_attention(q, k, v, "BSND", w.txt_len, w.latent, np.float32(w.sparsity))
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    finally:
        dist.destroy_process_group()
