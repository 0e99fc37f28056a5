"""GPU parity: dense attention and the reuse-step sparse kernel against the fp64 oracle.

The reuse kernel is fed the oracle's own metadata (grouping, KV indices,
residual rounded to bf16) so it is checked independently of the anchor kernels.
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import assert_close, f64, from_dev_bf16, oracle_metadata, to_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CASES = [  # (N, H, d, density, seed): several tiles, ragged N and K tails
    (4096, 2, 64, 0.25, 1001),
    (300, 2, 128, 0.26, 21),
    (1000, 1, 128, 0.333, 22),
    (777, 3, 64, 0.1, 23),
]


@pytest.fixture(scope="module")
def mcs():
    import free_sparse_attention_pddp_b200 as m

    m.load()
    return m


def _inputs(N, H, d, seed, step=0):
    w = synth.small(N, H=H, d=d, seed=seed)
    return w, synth.generate(w, "q", step), synth.generate(w, "k", step), synth.generate(w, "v", step)


@pytest.mark.parametrize("one_tile", [False, True], ids=["pair-kernel", "one-tile-kernel"])
@pytest.mark.parametrize("N,H,d,s,seed", CASES)
def test_dense_matches_oracle(mcs, N, H, d, s, seed, one_tile):
    """At d = 128 mcs_dense runs over pairs of query tiles (G odd in the 300-token
    case: the last pair has no second tile); debug flag bit 2 selects the
    one-tile kernel. d = 64 has only the one-tile kernel."""
    from free_sparse_attention_pddp_b200.binding import debug_set_flags

    w, q, k, v = _inputs(N, H, d, seed)
    shape = mcs.Shape(1, H, N, d)
    o = torch.empty(1, N, H, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(1, H, N, dtype=torch.float32, device="cuda")
    ws = mcs.workspace(shape, mcs.MCS_OP_DENSE)
    debug_set_flags(4 if one_tile else 0)
    try:
        mcs.mcs_dense(shape, to_dev(q), to_dev(k), to_dev(v), o, lse, ws)
        st, info = mcs.mcs_poll_status(ws)
    finally:
        debug_set_flags(0)
    assert st == 0, info
    got = f64(from_dev_bf16(o))
    rows = np.arange(N, dtype=np.int32)

    def one(h):
        return oracle.attention_rows(q, k, v, 0, h, rows)

    res = oracle.run_groups(one, range(H), threads=H)
    for h, (oref, lref) in enumerate(res):
        assert_close(got[0, :, h, :], oref, f"dense o head {h}")
        assert np.abs(lse.cpu().numpy()[0, h] - lref).max() < 2e-3


@pytest.mark.parametrize("N,H,d,s,seed", CASES[:2])
def test_dense_matches_torch_sdpa(mcs, N, H, d, s, seed):
    w, q, k, v = _inputs(N, H, d, seed)
    Q, K, V = (to_dev(t) for t in (q, k, v))
    shape = mcs.Shape(1, H, N, d)
    o = torch.empty_like(Q)
    ws = mcs.workspace(shape, mcs.MCS_OP_DENSE)
    mcs.mcs_dense(shape, Q, K, V, o, None, ws)
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q.float().transpose(1, 2), K.float().transpose(1, 2), V.float().transpose(1, 2)).transpose(1, 2)
    err = (o.float() - ref).abs()
    assert err.max().item() < 2e-2 and err.mean().item() < 2e-3


@pytest.mark.parametrize("N,H,d,s,seed", CASES)
def test_reuse_sparse_matches_oracle(mcs, N, H, d, s, seed):
    w, q0, k0, v0 = _inputs(N, H, d, seed, 0)
    _, q1, k1, v1 = _inputs(N, H, d, seed, 1)
    K = synth.topk_for(N, s)
    P, IDX, R, OD, LSE = oracle_metadata(q0, k0, v0, K)
    rb = oracle.round_bf16(R)
    shape = mcs.Shape(1, H, N, d, topk=K)
    o = torch.empty(1, N, H, d, dtype=torch.bfloat16, device="cuda")
    ws = mcs.workspace(shape, mcs.MCS_OP_SPARSE)
    dP, dI, dR = (torch.from_numpy(P).cuda(), torch.from_numpy(IDX).cuda(),
                  torch.from_numpy(rb.view(np.int16)).view(torch.bfloat16).cuda())
    mcs.mcs_sparse(shape, to_dev(q1), to_dev(k1), to_dev(v1), dP, dI, dR, o, ws)
    st, info = mcs.mcs_poll_status(ws)
    assert st == 0, info
    got = f64(from_dev_bf16(o))
    G = (N + 127) // 128
    for h in range(H):
        want = np.zeros((N, d))
        for g in range(G):
            rows = P[0, h, g * 128:(g + 1) * 128]
            want[rows] = oracle.reuse_group(q1, k1, v1, 0, h, rows, IDX[0, h, g],
                                            f64(rb[0, h, g * 128:g * 128 + len(rows)]))
        assert_close(got[0, :, h, :], want, f"reuse o head {h}")
    # no residual: plain token-sparse attention
    mcs.mcs_sparse(shape, to_dev(q1), to_dev(k1), to_dev(v1), dP, dI, None, o, ws)
    got = f64(from_dev_bf16(o))
    rows = P[0, 0, :128]
    want = oracle.reuse_group(q1, k1, v1, 0, 0, rows, IDX[0, 0, 0], None)
    assert_close(got[0, rows, 0, :], want, "sparse o without residual")
