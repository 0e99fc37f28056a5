"""Edge shapes through every call: a single token, one partial group, exactly
one group, one over a group, and a batch of two."""
import numpy as np
import pytest

import oracle
import synth
from helpers import assert_close, check_kv_idx_valid, f64, from_dev_bf16, to_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mcs():
    import free_sparse_attention_pddp_b200 as m

    m.load()
    return m


@pytest.mark.parametrize("B,N,H,d,K", [(1, 1, 1, 64, 1), (1, 127, 2, 128, 40), (1, 128, 1, 64, 128),
                                       (1, 129, 1, 128, 65), (2, 300, 2, 64, 77), (2, 640, 3, 128, 100)])
def test_whole_path_edges(mcs, B, N, H, d, K):
    w = synth.small(N, H=H, d=d, seed=N + B, B=B)
    q0, k0, v0 = (synth.generate(w, t, 0) for t in "qkv")
    q1, k1, v1 = (synth.generate(w, t, 1) for t in "qkv")
    G = (N + 127) // 128
    shape = mcs.Shape(B, H, N, d, topk=K)
    perm = torch.empty(B, H, N, dtype=torch.int32, device="cuda")
    idx = torch.empty(B, H, G, K, dtype=torch.int32, device="cuda")
    resid = torch.empty(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    o0 = torch.empty(B, N, H, d, dtype=torch.bfloat16, device="cuda")
    o1 = torch.empty_like(o0)
    ws = {op: mcs.workspace(shape, op) for op in (mcs.MCS_OP_GROUP, mcs.MCS_OP_ANCHOR, mcs.MCS_OP_SPARSE)}
    mcs.mcs_group(shape, to_dev(q0), perm, ws[mcs.MCS_OP_GROUP])
    mcs.mcs_anchor(shape, to_dev(q0), to_dev(k0), to_dev(v0), perm, o0, idx, resid, None, ws[mcs.MCS_OP_ANCHOR])
    mcs.mcs_sparse(shape, to_dev(q1), to_dev(k1), to_dev(v1), perm, idx, resid, o1, ws[mcs.MCS_OP_SPARSE])
    for wsx in ws.values():
        st, info = mcs.mcs_poll_status(wsx)
        assert st == 0, info
    P = perm.cpu().numpy()
    I = idx.cpu().numpy()
    check_kv_idx_valid(I, N, K)
    g0 = f64(from_dev_bf16(o0))
    g1 = f64(from_dev_bf16(o1))
    for b in range(B):
        for h in range(H):
            want_p, _ = oracle.pddp(q0, b, h)
            assert np.array_equal(P[b, h], want_p)
            for g in range(G):
                rows = want_p[g * 128:(g + 1) * 128]
                a = oracle.anchor_group(q0, k0, v0, b, h, rows, K)
                assert np.array_equal(I[b, h, g], a["idx"])
                assert_close(g0[b, rows, h], a["o_dense"], f"o_dense b{b} h{h} g{g}")
                o_ref = oracle.reuse_group(q1, k1, v1, b, h, rows, a["idx"], a["resid"])
                assert_close(g1[b, rows, h], o_ref, f"reuse b{b} h{h} g{g}")
