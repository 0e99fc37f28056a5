"""GPU parity of Fast PDDP grouping (mcs_group) against the fp64 oracle.

Every node of the grouping tree is replayed: the oracle splits the GPU's
member set and the two left children must agree, except for members whose
projection is within 1e-6 (relative) of the split value.
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import pddp_replay, to_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mcs():
    import free_sparse_attention_pddp_b200 as m

    m.load()
    return m


def _group(mcs, q):
    B, N, H, d = q.shape
    shape = mcs.Shape(B, H, N, d)
    perm = torch.full((B, H, N), -1, dtype=torch.int32, device="cuda")
    ws = mcs.workspace(shape, mcs.MCS_OP_GROUP)
    mcs.mcs_group(shape, to_dev(q), perm, ws)
    st, info = mcs.mcs_poll_status(ws)
    assert st == 0, info
    return perm.cpu().numpy()


@pytest.mark.parametrize("N,H,d,seed", [(4096, 2, 64, 1001), (1000, 2, 128, 41), (300, 1, 128, 42), (129, 1, 64, 43),
                                         (6000, 1, 128, 44)])
def test_group_matches_oracle(mcs, N, H, d, seed):
    w = synth.small(N, H=H, d=d, seed=seed)
    q = synth.generate(w, "q")
    perm = _group(mcs, q)
    for h in range(H):
        p = perm[0, h]
        assert np.array_equal(np.sort(p), np.arange(N))
        for gi in range(0, N, 128):
            assert np.all(np.diff(p[gi:gi + 128]) > 0)
        nodes, exact, tol, weak = pddp_replay(q, 0, h, p)
        assert weak == 0
        want, _ = oracle.pddp(q, 0, h)
        same = np.array_equal(p, want)
        print(f"N={N} h={h}: {nodes} nodes, {exact} exact, {tol} near-tie, full perm identical: {same}")
        if tol == 0:
            assert same


def _clustered_queries(N, d, gap, ncluster, seed):
    """Queries whose sample covariance has its top eigenvalue 1 just above a
    cluster of `ncluster` eigenvalues in [1 - 5 gap, 1 - gap] (before bf16
    rounding), the rest spread over [0.01, 0.81], in a random orientation."""
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((N, d))
    z -= z.mean(0)
    w, u = np.linalg.eigh(z.T @ z / N)
    z = z @ u @ np.diag(w ** -0.5) @ u.T  # sample covariance exactly the identity
    sig = np.linspace(0.9, 0.1, d)
    sig[0] = 1.0
    sig[1:1 + ncluster] = np.sqrt(np.linspace(1.0 - gap, 1.0 - 5 * gap, ncluster))
    rot, _ = np.linalg.qr(rng.standard_normal((d, d)))
    x = (z * sig) @ rot.T + 0.25
    bits = torch.from_numpy(x.astype(np.float32)).bfloat16().view(torch.int16).numpy().view(np.uint16)
    return bits.reshape(1, N, 1, d)


def test_group_small_eigengap_restarts(mcs):
    """A node whose top eigenvalue sits just above a tight cluster needs more
    Lanczos steps than one 64-vector cycle holds: the kernel restarts from its
    Ritz vector until the residual criterion holds, and the split still
    matches the oracle's (which takes the eigenvector from a full Jacobi
    eigensolver)."""
    N, d = 256, 128  # one internal node: the root
    q = _clustered_queries(N, d, 1e-3, 40, 9)
    shape = mcs.Shape(1, 1, N, d)
    perm = torch.full((1, 1, N), -1, dtype=torch.int32, device="cuda")
    ws = mcs.workspace(shape, mcs.MCS_OP_GROUP)
    mcs.mcs_group(shape, to_dev(q), perm, ws)
    st, info = mcs.mcs_poll_status(ws)
    assert st == 0, info
    assert info[6] == 1 and info[5] > 64, info  # one node; more than one cycle of steps
    p = perm.cpu().numpy()[0, 0]
    r = oracle.pddp_split(q, 0, 0, np.arange(N, dtype=np.int32), 128)
    gap = (r["eig"][0] - r["eig"][1]) / r["eig"][0]
    assert 1e-4 < gap < 2e-3, gap
    nodes, exact, tol, weak = pddp_replay(q, 0, 0, p)
    assert nodes == 1 and weak == 0 and exact + tol == 1
    print(f"relative eigengap {gap:.2e}: {info[5]} Lanczos steps, split {'exact' if exact else 'near-tie'}")


def test_group_rank1_sorts_by_latent(mcs):
    import torch as _t

    rng = np.random.default_rng(5)
    N, d = 640, 64
    u = rng.choice([-1.0, 1.0], size=d)
    u[3] *= 2.0
    pos = np.concatenate([np.arange(128, 256) / 2.0 ** s for s in range(4)])
    a = rng.permutation(np.concatenate([pos, -pos]))[:N]
    x = np.outer(a, u)[None, :, None, :].astype(np.float32)
    q = _t.from_numpy(x).to(_t.bfloat16).view(_t.int16).numpy().view(np.uint16)
    perm = _group(mcs, q)[0, 0]
    order = np.argsort(a * np.sign(u[3]), kind="stable")
    for gi in range(0, N, 128):
        assert np.array_equal(perm[gi:gi + 128], np.sort(order[gi:gi + 128]))


def _group_fast(mcs, q, k):
    B, N, H, d = q.shape
    shape = mcs.Shape(B, H, N, d)
    perm = torch.full((B, H, N), -1, dtype=torch.int32, device="cuda")
    ws = mcs.workspace(shape, mcs.MCS_OP_GROUP)
    mcs.mcs_group_fast(shape, to_dev(q), perm, k, ws)
    st, info = mcs.mcs_poll_status(ws)
    assert st == 0, info
    return perm.cpu().numpy()


def _krylov_replay(q, b, h, perm, k, rel=1e-6):
    """Every internal node: the oracle's k-step Krylov split of the GPU's member set must send the
    same members left, except members whose projection is within rel * max|p| of the split value."""
    exact = tolerated = 0
    for off, n, L in oracle.pddp_tree(perm.shape[0], 128):
        mem = np.sort(perm[off:off + n])
        r = oracle.pddp_split_krylov(q, b, h, mem, k)
        diff = set(map(int, perm[off:off + L])) ^ set(map(int, r["left"]))
        if not diff:
            exact += 1
            continue
        proj = dict(zip(map(int, mem), r["proj"]))
        pmax = np.abs(r["proj"]).max()
        for j in diff:
            assert abs(proj[j] - r["split_p"]) <= rel * pmax, f"node off={off} n={n}: token {j} (k={k})"
        tolerated += 1
    return exact, tolerated


@pytest.mark.parametrize("N,H,d,seed,k", [(1000, 2, 128, 41, 8), (4096, 1, 64, 1001, 4), (300, 1, 128, 42, 16),
                                           (6000, 1, 128, 44, 8), (777, 1, 64, 45, 2)])
def test_group_fast_matches_krylov_oracle(mcs, N, H, d, seed, k):
    w = synth.small(N, H=H, d=d, seed=seed)
    q = synth.generate(w, "q")
    perm = _group_fast(mcs, q, k)
    for h in range(H):
        p = perm[0, h]
        assert np.array_equal(np.sort(p), np.arange(N))
        for gi in range(0, N, 128):
            assert np.all(np.diff(p[gi:gi + 128]) > 0)
        exact, tol = _krylov_replay(q, 0, h, p, k)
        want = oracle.pddp_krylov(q, 0, h, k)
        print(f"N={N} h={h} k={k}: {exact} exact nodes, {tol} near-tie; full perm identical: "
              f"{np.array_equal(p, want)}")
        if tol == 0:
            assert np.array_equal(p, want)


def test_group_fast_full_space_is_the_exact_method(mcs):
    """k = d: the Krylov space is the whole space, so every split is the exact method's."""
    N, d = 1000, 64
    w = synth.small(N, H=1, d=d, seed=46)
    q = synth.generate(w, "q")
    p = _group_fast(mcs, q, d)[0, 0]
    nodes, exact, tol, weak = pddp_replay(q, 0, 0, p)
    assert weak == 0 and exact + tol == nodes


def test_group_fast_rank1_sorts_by_latent(mcs):
    import torch as _t

    rng = np.random.default_rng(5)
    N, d = 640, 64
    u = rng.choice([-1.0, 1.0], size=d)
    u[3] *= 2.0
    pos = np.concatenate([np.arange(128, 256) / 2.0 ** s for s in range(4)])
    a = rng.permutation(np.concatenate([pos, -pos]))[:N]
    q = _t.from_numpy(np.outer(a, u)[None, :, None, :].astype(np.float32)).to(_t.bfloat16).view(_t.int16).numpy()
    perm = _group_fast(mcs, q.view(np.uint16), 2)[0, 0]
    order = np.argsort(a * np.sign(u[3]), kind="stable")
    for gi in range(0, N, 128):
        assert np.array_equal(perm[gi:gi + 128], np.sort(order[gi:gi + 128]))


def test_group_fast_scatter_close_to_exact(mcs):
    """Within-group scatter (the quantity the grouping minimises) of the fast grouping stays close to
    the exact method's and far below token order's."""
    N, d = 6000, 128
    w = synth.small(N, H=1, d=d, seed=47)
    q = synth.generate(w, "q")
    x = synth.bf16_to_f64(q)[0, :, 0, :]

    def scatter(p):
        return sum(((x[p[i:i + 128]] - x[p[i:i + 128]].mean(0)) ** 2).sum() for i in range(0, N, 128))

    s_exact = scatter(_group(mcs, q)[0, 0])
    s_ident = scatter(np.arange(N))
    for k in (4, 8, 16):
        s_fast = scatter(_group_fast(mcs, q, k)[0, 0])
        print(f"k={k}: scatter fast/exact {s_fast / s_exact:.4f}, token order/exact {s_ident / s_exact:.3f}")
        assert s_fast <= 1.05 * s_exact
    assert s_ident > 1.2 * s_exact


def test_group_fast_arguments(mcs):
    shape = mcs.Shape(1, 1, 256, 64)
    ws = mcs.workspace(shape, mcs.MCS_OP_GROUP)
    q = torch.zeros(1, 256, 1, 64, dtype=torch.bfloat16, device="cuda")
    perm = torch.empty(1, 1, 256, dtype=torch.int32, device="cuda")
    for k in (1, 0, 65):
        with pytest.raises(mcs.MCSError):
            mcs.mcs_group_fast(shape, q, perm, k, ws)


def _group_ex(mcs, q, krylov=0, whiten=True):
    B, N, H, d = q.shape
    shape = mcs.Shape(B, H, N, d)
    perm = torch.full((B, H, N), -1, dtype=torch.int32, device="cuda")
    ws = mcs.workspace(shape, mcs.MCS_OP_GROUP)
    mcs.mcs_group_ex(shape, to_dev(q), perm, ws, krylov_steps=krylov, whiten=whiten)
    st, info = mcs.mcs_poll_status(ws)
    assert st == 0, info
    return perm.cpu().numpy()


def _channel_scaled(q, seed):
    """The same queries with channel c multiplied by a power of two (exact in bf16), so that
    per-channel standardisation changes the grouping."""
    k = np.random.default_rng(seed).integers(-3, 4, q.shape[-1])
    x = synth.bf16_to_f64(q) * 2.0 ** k
    out = (x.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(synth.bf16_to_f64(out), x)
    return out


@pytest.mark.parametrize("N,H,d,seed", [(1000, 2, 128, 51), (700, 1, 64, 52), (4096, 1, 64, 1001),
                                         (6000, 1, 128, 53)])
def test_group_whitened_matches_oracle(mcs, N, H, d, seed):
    """Whitened grouping (mcs_group_ex, MCS_GROUP_WHITEN) node by node against the oracle's
    PDDP on the per-channel standardised queries."""
    w = synth.small(N, H=H, d=d, seed=seed)
    q = _channel_scaled(synth.generate(w, "q"), seed)
    perm = _group_ex(mcs, q)
    plain = _group(mcs, q)
    for h in range(H):
        p = perm[0, h]
        assert np.array_equal(np.sort(p), np.arange(N))
        ws = oracle.channel_scale(q, 0, h)
        nodes, exact, tol, weak = pddp_replay(q, 0, h, p, wscale=ws)
        assert weak == 0
        want = oracle.pddp_whitened(q, 0, h)
        if tol == 0:
            assert np.array_equal(p, want)
        assert not np.array_equal(p, plain[0, h])  # the channel scales matter here
        print(f"whitened N={N} h={h}: {nodes} nodes, {exact} exact, {tol} near-tie")


def test_group_whitened_is_channel_scale_invariant(mcs):
    """Scaling channels by powers of two leaves the whitened queries, and so the whitened grouping,
    unchanged, for the converged and the fixed-step directions alike."""
    w = synth.small(2000, H=2, d=128, seed=57)
    q = synth.generate(w, "q")
    q2 = _channel_scaled(q, 58)
    for krylov in (0, 8):
        assert np.array_equal(_group_ex(mcs, q, krylov), _group_ex(mcs, q2, krylov))


def test_group_ex_arguments(mcs):
    shape = mcs.Shape(1, 1, 256, 64)
    x = torch.zeros(1, 256, 1, 64, dtype=torch.bfloat16, device="cuda")
    perm = torch.empty(1, 1, 256, dtype=torch.int32, device="cuda")
    ws = mcs.workspace(shape, mcs.MCS_OP_GROUP)
    for kw in (dict(krylov_steps=1), dict(krylov_steps=65)):
        with pytest.raises(mcs.MCSError) as e:
            mcs.mcs_group_ex(shape, x, perm, ws, **kw)
        assert e.value.code == 1
    lib = mcs.load()
    import ctypes
    rc = lib.mcs_group_ex(ctypes.byref(shape), ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(perm.data_ptr()), 0,
                          2, ctypes.c_void_p(ws.data_ptr()), ws.numel(), None)
    assert rc == 1  # unknown flag bit
