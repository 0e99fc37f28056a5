"""Ulysses exchanges (seq_to_heads / heads_to_seq) on 2 to 7 gloo ranks, on CPU.

The exchanges are the only multi-rank step of head-parallel MC-Sparse. Each
rank holds a sequence shard of Q, K, V; after seq_to_heads it holds every token
of its heads, a per-head attention runs there, and heads_to_seq returns the
rank's sequence shard of the output. Checked: the head shard is exactly the
slice of the full tensor, the round trip is the identity, and the composition
with per-head attention equals attention on the unsharded tensors -- also on
7 ranks with 24 and 40 heads (the pages' 7 denoising GPUs with the MiniMax-H3
and Wan-14B head counts, which do not divide by 7), with a sequence length
that does not divide either, and with more ranks than heads.
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
        from free_sparse_attention_pddp_b200.ulysses import heads_to_seq, seq_to_heads, split_counts

        g = torch.Generator().manual_seed(123)
        q, k, v = (torch.randn(B, N, H, d, generator=g, dtype=torch.float64) for _ in range(3))
        nr, hr = split_counts(N, world), split_counts(H, world)
        r0, h0 = sum(nr[:rank]), sum(hr[:rank])
        rows = slice(r0, r0 + nr[rank])
        heads = slice(h0, h0 + hr[rank])
        qh = seq_to_heads(q[:, rows].contiguous(), N=N)
        assert qh.shape == (B, N, hr[rank], d)
        assert torch.equal(qh, q[:, :, heads])
        assert torch.equal(heads_to_seq(qh, H=H), q[:, rows])
        kh, vh = (seq_to_heads(t[:, rows].contiguous(), N=N) for t in (k, v))
        oh = _attention(qh, kh, vh) if hr[rank] > 0 else torch.empty_like(qh)
        o = heads_to_seq(oh, H=H)
        want = _attention(q, k, v)[:, rows]
        assert torch.allclose(o, want, rtol=0, atol=1e-12)
        dist.destroy_process_group()
    except Exception as exc:  # reported to the parent
        errq.put(f"rank {rank}: {type(exc).__name__}: {exc}")
        raise


@pytest.mark.parametrize("world,B,N,H,d", [(2, 1, 64, 4, 8), (4, 2, 96, 8, 4), (2, 1, 10, 2, 16),
                                           (7, 1, 70, 24, 8), (7, 1, 75, 40, 4), (3, 2, 11, 2, 4)])
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


def test_split_counts():
    from free_sparse_attention_pddp_b200.ulysses import split_counts

    assert split_counts(24, 7) == [4, 4, 4, 3, 3, 3, 3]
    assert split_counts(40, 7) == [6, 6, 6, 6, 6, 5, 5]
    assert split_counts(87696, 7) == [12528] * 7
    assert split_counts(2, 3) == [1, 1, 0]
    assert sum(split_counts(75601, 8)) == 75601
    with pytest.raises(ValueError):
        split_counts(5, 0)


def test_shard_of_the_wrong_size_is_rejected():
    from free_sparse_attention_pddp_b200 import ulysses

    orig_w, orig_r = ulysses._world, ulysses._rank
    ulysses._world, ulysses._rank = (lambda group: 2), (lambda group: 1)
    try:
        with pytest.raises(ValueError):  # 11 tokens over 2 ranks: rank 1 holds 5, not 6
            ulysses.seq_to_heads(torch.zeros(1, 6, 3, 2), N=11)
        with pytest.raises(ValueError):  # 3 heads over 2 ranks: rank 1 holds 1, not 2
            ulysses.heads_to_seq(torch.zeros(1, 5, 2, 2), H=3)
    finally:
        ulysses._world, ulysses._rank = orig_w, orig_r
