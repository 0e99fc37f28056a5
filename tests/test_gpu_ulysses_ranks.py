"""GPU: head-parallel MC-Sparse on two ranks with an uneven head split.

Two processes share the one GPU; their exchanges (seq_to_heads, heads_to_seq)
run over a gloo group on host copies of the shards, and each rank runs
grouping, anchor and reuse step through the C ABI on the heads it owns (3
heads over 2 ranks: 2 and 1; a sequence of 1001 tokens: 501 and 500 rows). The
ranks' kernels never wait on each other: each rank's calls are independent.
Every rank's anchor and reuse output shard must equal, bit for bit, the same
rows of direct calls over all heads in one process, since MC-Sparse is
independent per head.
"""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

N, H, D, DENSITY = 1001, 3, 64, 0.25


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _path(mcs, q0, k0, v0, q1, k1, v1, K):
    """Grouping, anchor and reuse on [1, N, h, D] device tensors: (anchor o, reuse o)."""
    B, n, h, d = q0.shape
    shape = mcs.Shape(B, h, n, d, topk=K)
    ws = {op: mcs.workspace(shape, op) for op in (mcs.MCS_OP_GROUP, mcs.MCS_OP_ANCHOR, mcs.MCS_OP_SPARSE)}
    perm = torch.empty(B, h, n, dtype=torch.int32, device="cuda")
    idx = torch.empty(B, h, (n + 127) // 128, K, dtype=torch.int32, device="cuda")
    resid = torch.empty(B, h, n, d, dtype=torch.bfloat16, device="cuda")
    oa, o1 = torch.empty_like(q0), torch.empty_like(q0)
    mcs.mcs_group(shape, q0, perm, ws[mcs.MCS_OP_GROUP])
    mcs.mcs_anchor(shape, q0, k0, v0, perm, oa, idx, resid, None, ws[mcs.MCS_OP_ANCHOR])
    mcs.mcs_sparse(shape, q1, k1, v1, perm, idx, resid, o1, ws[mcs.MCS_OP_SPARSE])
    for w in ws.values():
        assert mcs.mcs_poll_status(w)[0] == 0
    return oa, o1


def _worker(rank, world, port, errq):
    try:
        import numpy as np
        import torch.distributed as dist

        import free_sparse_attention_pddp_b200 as mcs
        import synth
        from free_sparse_attention_pddp_b200.ulysses import heads_to_seq, seq_to_heads, split_counts

        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        torch.cuda.set_device(0)
        mcs.load()
        w = synth.small(N, H=H, d=D, seed=91)
        K = synth.topk_for(N, DENSITY)
        host = {(t, s): torch.from_numpy(synth.generate(w, t, s).view(np.int16)).view(torch.bfloat16)
                for t in "qkv" for s in (0, 1)}
        rows = split_counts(N, world)
        r0 = sum(rows[:rank])
        # this rank's sequence shard -> every token of its heads (host exchange), then the GPU path
        shard = {key: x[:, r0:r0 + rows[rank]].contiguous() for key, x in host.items()}
        heads = {key: seq_to_heads(x, N=N).cuda() for key, x in shard.items()}
        oa_h, o1_h = _path(mcs, *(heads[(t, 0)] for t in "qkv"), *(heads[(t, 1)] for t in "qkv"), K)
        oa = heads_to_seq(oa_h.cpu(), H=H)
        o1 = heads_to_seq(o1_h.cpu(), H=H)
        # direct calls over all heads in this process
        full = {key: x.cuda() for key, x in host.items()}
        fa, f1 = _path(mcs, *(full[(t, 0)] for t in "qkv"), *(full[(t, 1)] for t in "qkv"), K)
        sl = slice(r0, r0 + rows[rank])
        assert torch.equal(oa.view(torch.int16), fa[:, sl].cpu().view(torch.int16)), "anchor output"
        assert torch.equal(o1.view(torch.int16), f1[:, sl].cpu().view(torch.int16)), "reuse output"
        dist.destroy_process_group()
    except Exception as exc:  # reported to the parent
        errq.put(f"rank {rank}: {type(exc).__name__}: {exc}")
        raise


def test_two_ranks_uneven_heads_equal_direct_calls():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    errq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, errq)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
    errs = []
    while not errq.empty():
        errs.append(errq.get())
    for p in procs:
        if p.is_alive():
            p.kill()
            errs.append("a rank did not finish")
    assert not errs and all(p.exitcode == 0 for p in procs), errs
