"""GPU parity of the anchor step (dense + lse, exact-probability group mass,
token-level top-K, sparse pass and residual) against the fp64 oracle.

The anchor is fed the oracle's grouping so that it is checked on its own.
KV indices must match the oracle's exactly except at near ties of the K-th
largest group mass (relative gap below 1e-6).
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import (assert_close, check_kv_idx_valid, f64, from_dev_bf16, index_mismatches_ok, oracle_metadata,
                     to_dev)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CASES = [  # (N, H, d, density, seed)
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
    return synth.generate(w, "q", step), synth.generate(w, "k", step), synth.generate(w, "v", step)


def _run_anchor(mcs, q, k, v, P, K):
    B, N, H, d = q.shape
    G = (N + 127) // 128
    shape = mcs.Shape(B, H, N, d, topk=K)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    o = torch.empty_like(dq)
    idx = torch.full((B, H, G, K), -1, dtype=torch.int32, device="cuda")
    resid = torch.empty(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
    ws = mcs.workspace(shape, mcs.MCS_OP_ANCHOR)
    dP = torch.from_numpy(P).cuda()
    mcs.mcs_anchor(shape, dq, dk, dv, dP, o, idx, resid, lse, ws)
    st, info = mcs.mcs_poll_status(ws)
    return dict(shape=shape, q=dq, k=dk, v=dv, P=dP, o=o, idx=idx, resid=resid, lse=lse, ws=ws, st=st, info=info)


@pytest.mark.parametrize("N,H,d,s,seed", CASES)
def test_anchor_matches_oracle(mcs, N, H, d, s, seed):
    q, k, v = _inputs(N, H, d, seed)
    K = synth.topk_for(N, s)
    P = np.stack([oracle.pddp(q, 0, h)[0] for h in range(H)])[None]
    r = _run_anchor(mcs, q, k, v, P, K)
    assert r["st"] == 0, r["info"]
    assert r["info"][2] == 0, "uncertain band overflowed"
    got_o = f64(from_dev_bf16(r["o"]))
    got_idx = r["idx"].cpu().numpy()
    got_r = f64(from_dev_bf16(r["resid"]))
    got_lse = r["lse"].cpu().numpy()
    check_kv_idx_valid(got_idx, N, K)
    G = (N + 127) // 128
    mism = 0
    for h in range(H):
        want_o = np.zeros((N, d))
        res = oracle.run_groups(lambda g: oracle.anchor_group(q, k, v, 0, h, P[0, h, g * 128:(g + 1) * 128], K),
                                range(G), threads=8)
        for g, a in enumerate(res):
            rows = P[0, h, g * 128:(g + 1) * 128]
            want_o[rows] = a["o_dense"]
            assert np.abs(got_lse[0, h, rows] - a["lse"]).max() < 2e-3
            n_mis, n_bad = index_mismatches_ok(got_idx[0, h, g], a["idx"], a["mass"], K)
            assert n_bad == 0, f"head {h} group {g}: {n_bad} KV indices differ beyond near ties"
            mism += n_mis
            if n_mis == 0:
                assert_close(got_r[0, h, g * 128:g * 128 + len(rows)], a["resid"], f"resid h{h} g{g}")
        assert_close(got_o[0, :, h, :], want_o, f"anchor o head {h}")
    print(f"near-tie index mismatches: {mism}; fp64-refined keys: {r['info'][3]}")


def test_anchor_sparse_plus_residual_is_dense(mcs):
    """At the anchor, reuse with unchanged Q/K/V reproduces the dense output (up to bf16 rounding of R)."""
    N, H, d = 1000, 2, 128
    q, k, v = _inputs(N, H, d, 31)
    K = 300
    P = np.stack([oracle.pddp(q, 0, h)[0] for h in range(H)])[None]
    r = _run_anchor(mcs, q, k, v, P, K)
    assert r["st"] == 0
    o2 = torch.empty_like(r["o"])
    ws = mcs.workspace(r["shape"], mcs.MCS_OP_SPARSE)
    mcs.mcs_sparse(r["shape"], r["q"], r["k"], r["v"], r["P"], r["idx"], r["resid"], o2, ws)
    a, b = r["o"].float(), o2.float()
    rmax = r["resid"].float().abs().max().item()
    assert (a - b).abs().max().item() <= 2 ** -8 * max(1.0, a.abs().max().item()) + 2 ** -8 * rmax


def test_anchor_full_density_zero_residual(mcs):
    N, H, d = 384, 1, 64
    q, k, v = _inputs(N, H, d, 32)
    P = oracle.pddp(q, 0, 0)[0][None, None]
    r = _run_anchor(mcs, q, k, v, P, N)
    assert r["st"] == 0
    idx = r["idx"].cpu().numpy()
    assert np.array_equal(idx[0, 0], np.broadcast_to(np.arange(N), (3, N)))
    # O_dense and O_sparse are both convex combinations of the V rows with the
    # same exact weights up to the bf16 rounding of each probability (2^-9
    # relative, renormalised by an fp32 sum): each is within 2 * 2^-9 * max|V|
    # of the exact output, so R = O_dense - O_sparse is within 2^-7 * max|V|.
    # (The dense pass and the sparse pass round P at different running maxima.)
    vmax = float(np.abs(f64(v)).max())
    assert r["resid"].float().abs().max().item() <= 2 ** -7 * vmax


def test_anchor_k1_selects_argmax_and_value_row(mcs):
    N, H, d = 512, 1, 128
    q, k, v = _inputs(N, H, d, 33)
    P = oracle.pddp(q, 0, 0)[0][None, None]
    r = _run_anchor(mcs, q, k, v, P, 1)
    assert r["st"] == 0
    idx = r["idx"].cpu().numpy()[0, 0, :, 0]
    o2 = torch.empty_like(r["o"])
    ws = mcs.workspace(r["shape"], mcs.MCS_OP_SPARSE)
    mcs.mcs_sparse(r["shape"], r["q"], r["k"], r["v"], r["P"], r["idx"], None, o2, ws)
    got = from_dev_bf16(o2)
    for g in range(4):
        rows = P[0, 0, g * 128:(g + 1) * 128]
        m = oracle.group_mass(q, k, 0, 0, rows)
        assert idx[g] == int(np.argmax(m))
        assert np.array_equal(got[0, rows, 0, :], np.repeat(v[0, idx[g]:idx[g] + 1, 0, :], len(rows), axis=0))


def test_anchor_then_reuse_matches_oracle(mcs):
    """Anchor on step 0 (GPU), reuse on step 1 (GPU) vs the oracle's anchor + reuse."""
    N, H, d, s, seed = 4096, 2, 64, 0.25, 1001
    w = synth.WORKLOADS["tiny"]
    q0, k0, v0 = (synth.generate(w, t, 0) for t in "qkv")
    q1, k1, v1 = (synth.generate(w, t, 1) for t in "qkv")
    K = w.topk
    P = np.stack([oracle.pddp(q0, 0, h)[0] for h in range(H)])[None]
    r = _run_anchor(mcs, q0, k0, v0, P, K)
    assert r["st"] == 0
    o = torch.empty_like(r["o"])
    ws = mcs.workspace(r["shape"], mcs.MCS_OP_SPARSE)
    mcs.mcs_sparse(r["shape"], to_dev(q1), to_dev(k1), to_dev(v1), r["P"], r["idx"], r["resid"], o, ws)
    got = f64(from_dev_bf16(o))
    _, IDX, R, _, _ = oracle_metadata(q0, k0, v0, K, perm=P[0][None] if P.ndim == 3 else P)
    for h in range(H):
        want = np.zeros((N, d))
        for g in range(N // 128):
            rows = P[0, h, g * 128:(g + 1) * 128]
            want[rows] = oracle.reuse_group(q1, k1, v1, 0, h, rows, IDX[0, h, g], R[0, h, g * 128:(g + 1) * 128])
        assert_close(got[0, :, h, :], want, f"anchor+reuse head {h}")


TOPK_PATH_CASES = [  # (N, H, d, density, seed, zero_q)
    (4096, 2, 64, 0.25, 1001, False),
    (777, 3, 64, 0.1, 23, False),
    (9000, 1, 128, 0.2, 24, False),
    (1000, 1, 128, 0.3, 25, True),   # every mass equal: ties resolved by index in the band
    (3000, 1, 64, 0.3, 26, True),    # every mass equal, band wider than its buffer: fp32 ranking
]


@pytest.mark.parametrize("N,H,d,s,seed,zero_q", TOPK_PATH_CASES)
def test_topk_two_sweep_path_matches_general_path(mcs, N, H, d, s, seed, zero_q):
    """The two-sweep top-K and the general seven-sweep one (forced by test hook bit 1) select the same keys."""
    q, k, v = _inputs(N, H, d, seed)
    if zero_q:
        q = np.zeros_like(q)
    K = synth.topk_for(N, s)
    P = np.stack([np.arange(N, dtype=np.int32)] * H)[None]
    G = (N + 127) // 128
    from free_sparse_attention_pddp_b200.binding import debug_set_flags

    runs = []
    try:
        for flags in (0, 2):
            debug_set_flags(flags)
            r = _run_anchor(mcs, q, k, v, P, K)
            assert r["st"] == 0, r["info"]
            runs.append(r)
    finally:
        debug_set_flags(0)
    fast, full = runs
    assert full["info"][4] == H * G  # every group took the general path
    if not zero_q:
        assert fast["info"][4] <= max(1, H * G // 20), fast["info"]  # the general path stays rare
    check_kv_idx_valid(fast["idx"].cpu().numpy(), N, K)
    assert torch.equal(fast["idx"], full["idx"])
    assert torch.equal(fast["resid"].view(torch.int16), full["resid"].view(torch.int16))
    assert fast["info"][2] == full["info"][2] and fast["info"][3] == full["info"][3]
