"""GPU: UlyssesMCSparse on a one-rank NCCL group equals the direct library calls.

With one rank the two all-to-alls are identities, so the wrapper's anchor and
reuse outputs (and its cached metadata) must equal, bit for bit, mcs_group +
mcs_anchor and mcs_sparse run directly on the same tensors. The multi-rank
exchanges are covered on CPU with gloo ranks (tests/test_ulysses_cpu.py).
"""
import os
import socket

import pytest

import synth
from helpers import to_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nccl_group():
    import torch.distributed as dist

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta

    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    yield
    dist.destroy_process_group()


def test_one_rank_wrapper_equals_direct_calls(nccl_group):
    import free_sparse_attention_pddp_b200 as mcs
    from free_sparse_attention_pddp_b200.ulysses import UlyssesMCSparse

    N, H, d, s = 1000, 2, 128, 0.25
    w = synth.small(N, H=H, d=d, seed=61)
    q0, k0, v0 = (to_dev(synth.generate(w, t, 0)) for t in "qkv")
    q1, k1, v1 = (to_dev(synth.generate(w, t, 1)) for t in "qkv")
    K = synth.topk_for(N, s)
    for krylov in (0, 8):
        u = UlyssesMCSparse(1, H, N, d, K, krylov_steps=krylov)
        oa = u.anchor(q0, k0, v0)
        ore = u.reuse(q1, k1, v1)
        assert not u.status()
        shape = mcs.Shape(1, H, N, d, topk=K)
        ws = {op: mcs.workspace(shape, op) for op in (mcs.MCS_OP_GROUP, mcs.MCS_OP_ANCHOR, mcs.MCS_OP_SPARSE)}
        perm = torch.empty_like(u.perm)
        idx = torch.empty_like(u.kv_idx)
        resid = torch.empty_like(u.resid)
        if krylov:
            mcs.mcs_group_fast(shape, q0, perm, krylov, ws[mcs.MCS_OP_GROUP])
        else:
            mcs.mcs_group(shape, q0, perm, ws[mcs.MCS_OP_GROUP])
        o0 = torch.empty_like(q0)
        mcs.mcs_anchor(shape, q0, k0, v0, perm, o0, idx, resid, None, ws[mcs.MCS_OP_ANCHOR])
        o1 = torch.empty_like(q1)
        mcs.mcs_sparse(shape, q1, k1, v1, perm, idx, resid, o1, ws[mcs.MCS_OP_SPARSE])
        torch.cuda.synchronize()
        assert torch.equal(u.perm, perm) and torch.equal(u.kv_idx, idx)
        assert torch.equal(u.resid.view(torch.int16), resid.view(torch.int16))
        assert torch.equal(oa.view(torch.int16), o0.view(torch.int16))
        assert torch.equal(ore.view(torch.int16), o1.view(torch.int16))


def test_reuse_before_anchor_raises(nccl_group):
    from free_sparse_attention_pddp_b200.ulysses import UlyssesMCSparse

    u = UlyssesMCSparse(1, 2, 256, 64, 32)
    q = torch.zeros(1, 256, 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(RuntimeError):
        u.reuse(q, q, q)
