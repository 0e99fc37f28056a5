"""Ulysses exchanges (seq_to_heads / heads_to_seq) on 2 and 4 gloo ranks, on CPU.

The exchanges are the only multi-rank step of head-parallel MC-Sparse. Each
rank holds a sequence shard of Q, K, V; after seq_to_heads it holds every token
of its heads, a per-head attention runs there, and heads_to_seq returns the
rank's sequence shard of the output. Checked: the head shard is exactly the
slice of the full tensor, the round trip is the identity, and the composition
with per-head attention equals attention on the unsharded tensors.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _attention(q, k, v):
    # plain per-head softmax attention in fp64 on [B, N, h, d]
    s = torch.einsum("bnhd,bmhd->bhnm", q, k) / q.shape[-1] ** 0.5
    return torch.einsum("bhnm,bmhd->bnhd", torch.softmax(s, dim=-1), v)


def _worker(rank, world, port, B, N, H, d, errq):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        from free_sparse_attention_pddp_b200.ulysses import heads_to_seq, seq_to_heads

        g = torch.Generator().manual_seed(123)
        q, k, v = (torch.randn(B, N, H, d, generator=g, dtype=torch.float64) for _ in range(3))
        n, hp = N // world, H // world
        rows = slice(rank * n, (rank + 1) * n)
        heads = slice(rank * hp, (rank + 1) * hp)
        qh = seq_to_heads(q[:, rows].contiguous())
        assert torch.equal(qh, q[:, :, heads])
        assert torch.equal(heads_to_seq(qh), q[:, rows])
        oh = _attention(qh, seq_to_heads(k[:, rows].contiguous()), seq_to_heads(v[:, rows].contiguous()))
        o = heads_to_seq(oh)
        want = _attention(q, k, v)[:, rows]
        assert torch.allclose(o, want, rtol=0, atol=1e-12)
        dist.destroy_process_group()
    except Exception as exc:  # reported to the parent
        errq.put(f"rank {rank}: {type(exc).__name__}: {exc}")
        raise


@pytest.mark.parametrize("world,B,N,H,d", [(2, 1, 64, 4, 8), (4, 2, 96, 8, 4), (2, 1, 10, 2, 16)])
def test_ulysses_exchanges_compose_with_per_head_attention(world, B, N, H, d):
    ctx = mp.get_context("spawn")
    errq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, B, N, H, d, errq)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    errs = []
    while not errq.empty():
        errs.append(errq.get())
    for p in procs:
        if p.is_alive():
            p.kill()
            errs.append("a rank did not finish")
    assert not errs and all(p.exitcode == 0 for p in procs), errs


def test_uneven_split_is_rejected():
    from free_sparse_attention_pddp_b200 import ulysses

    x = torch.zeros(1, 4, 3, 2)  # 3 heads over 2 ranks
    orig = ulysses._world
    ulysses._world = lambda group: 2
    try:
        with pytest.raises(ValueError):
            ulysses.seq_to_heads(x)
        with pytest.raises(ValueError):
            ulysses.heads_to_seq(torch.zeros(1, 5, 2, 2))
    finally:
        ulysses._world = orig
