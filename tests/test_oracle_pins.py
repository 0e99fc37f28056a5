"""Pins for the fp64 CPU oracle: each check ties the oracle to something other
than itself (a library routine on a case that reduces to it, a closed form, an
invariant, brute force, or a number printed in the pages).

Every check is a plain function taking the oracle library handle, so the
mutation test can run the same checks against copies of the oracle with a
planted mistake and confirm that at least one check fails for each.
"""
import itertools
import math
import os

import numpy as np

import oracle
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bits(x):
    """float64 -> bf16 bits via torch's round-to-nearest-even (independent of the oracle)."""
    import torch

    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(
        np.uint16)


def _wide(bits):
    return synth.bf16_to_f64(bits)


def _tiny_qkv(N=256, H=1, d=32, seed=3):
    w = synth.small(N, H=H, d=d, seed=seed)
    return w, synth.generate(w, "q"), synth.generate(w, "k"), synth.generate(w, "v")


# ---------------------------------------------------------------------------
# eigen-solver
# ---------------------------------------------------------------------------

def check_jacobi_vs_numpy(lib):
    rng = np.random.default_rng(11)
    for n in (2, 7, 32, 64):
        A = rng.standard_normal((n, n))
        A = A + A.T
        ev, V, sweeps = oracle.jacobi_eigh(A, lib=lib)
        assert sweeps >= 0
        w, U = np.linalg.eigh(A)
        assert np.allclose(ev, w[::-1], atol=1e-10 * np.abs(w).max())
        # A V = V diag(ev) and V orthonormal
        assert np.allclose(A @ V, V * ev, atol=1e-9 * np.abs(w).max())
        assert np.allclose(V.T @ V, np.eye(n), atol=1e-11)
        # top eigenvector equal to numpy's up to sign
        top = U[:, -1]
        assert min(np.abs(V[:, 0] - top).max(), np.abs(V[:, 0] + top).max()) < 1e-8


def check_jacobi_2x2_closed_form(lib):
    for a, b, c in [(3.0, 1.0, -2.0), (1.0, 0.0, 1.0), (0.5, -4.0, 0.25), (2.0, 1e-9, 2.0)]:
        ev, V, _ = oracle.jacobi_eigh(np.array([[a, b], [b, c]]), lib=lib)
        mid, rad = (a + c) / 2, math.hypot((a - c) / 2, b)
        assert abs(ev[0] - (mid + rad)) < 1e-12 and abs(ev[1] - (mid - rad)) < 1e-12


def test_jacobi_vs_numpy(orc):
    check_jacobi_vs_numpy(orc)


def test_jacobi_2x2_closed_form(orc):
    check_jacobi_2x2_closed_form(orc)


# ---------------------------------------------------------------------------
# PDDP grouping
# ---------------------------------------------------------------------------

def _rank1(N, d, seed):
    """q_i = a_i * u with u = +-1 entries except one +-2, and distinct integer a_i: every value exact in bf16."""
    rng = np.random.default_rng(seed)
    u = rng.choice([-1.0, 1.0], size=d)
    u[seed % d] *= 2.0  # a unique largest-magnitude entry fixes the orientation rule unambiguously
    # distinct latents with 8-bit significands (m / 2^s, m in [128, 255]) so a*u is exact in bf16
    pos = np.concatenate([np.arange(128, 256) / 2.0 ** s for s in range(4)])
    a = rng.permutation(np.concatenate([pos, -pos]))[:N]
    q = np.outer(a, u)[None, :, None, :]
    return _bits(q), a, u


def check_pddp_rank1_sorts_by_latent(lib):
    for N, d in ((512, 16), (600, 32), (1000, 8)):
        q, a, u = _rank1(N, d, seed=N)
        perm, gaps = oracle.pddp(q, 0, 0, 128, lib=lib)
        # direction is +-u/|u|; the sign rule makes its largest-magnitude entry positive
        order = np.argsort(a * np.sign(u[N % d]), kind="stable")
        for gi in range(0, N, 128):
            assert np.array_equal(perm[gi:gi + 128], np.sort(order[gi:gi + 128])), (N, gi)
        assert np.all(gaps > 0.999)


def check_pddp_matches_numpy_projection(lib):
    """Every split equals a sort by projection on numpy eigh's principal direction (sign rule applied)."""
    # N = 700 is 6 tiles: both children of the root have an odd tile count
    w, q, _, _ = _tiny_qkv(N=700, d=32, seed=5)
    perm, gaps = oracle.pddp(q, 0, 0, 128, lib=lib)
    X = _wide(q[0, :, 0, :])
    assert np.array_equal(np.sort(perm), np.arange(700))
    for off, n, L in oracle.pddp_tree(700, 128):
        mem = np.sort(perm[off:off + n])
        Y = X[mem]
        mu = Y.mean(axis=0)
        C = (Y - mu).T @ (Y - mu)
        ev, U = np.linalg.eigh(C)
        v = U[:, -1]
        v = v * (1.0 if v[np.argmax(np.abs(v))] > 0 else -1.0)
        p = (Y - mu) @ v
        want_left = np.sort(mem[np.lexsort((mem, p))[:L]])
        assert np.array_equal(np.sort(perm[off:off + L]), want_left), (off, n)
        assert (ev[-1] - ev[-2]) / ev[-1] > 1e-3


def check_pddp_sizes_and_leaves(lib):
    for N in (128, 129, 256, 300, 640, 1000):
        _, q, _, _ = _tiny_qkv(N=N, d=16, seed=N)
        perm, _ = oracle.pddp(q, 0, 0, 128, lib=lib)
        assert np.array_equal(np.sort(perm), np.arange(N))
        for gi in range(0, N, 128):
            grp = perm[gi:gi + 128]
            assert len(grp) == min(128, N - gi)
            assert np.all(np.diff(grp) > 0)


def test_pddp_rank1_sorts_by_latent(orc):
    check_pddp_rank1_sorts_by_latent(orc)


def test_pddp_matches_numpy_projection(orc):
    check_pddp_matches_numpy_projection(orc)


def test_pddp_sizes_and_leaves(orc):
    check_pddp_sizes_and_leaves(orc)


def test_pddp_tree_shape():
    # T = 591 tiles (N = 75600) gives 10 levels, left children always whole tiles
    nodes = oracle.pddp_tree(75600, 128)
    assert len(nodes) == 590
    assert all(L % 128 == 0 and n - L > 0 for _, n, L in nodes)
    # one partial leaf, last in depth-first order
    leaves = []

    def rec(off, n):
        if (n + 127) // 128 <= 1:
            leaves.append((off, n))
            return
        L = oracle.pddp_left_size(n, 128)
        rec(off, L)
        rec(off + L, n - L)

    rec(0, 75600)
    assert [n for _, n in leaves[:-1]] == [128] * 590 and leaves[-1] == (75520, 80)


# ---------------------------------------------------------------------------
# dense attention, LSE, mass
# ---------------------------------------------------------------------------

def check_dense_vs_numpy(lib):
    from scipy.special import logsumexp

    w, q, k, v = _tiny_qkv(N=200, d=32, seed=9)
    Q, K, V = (_wide(t[0, :, 0, :]) for t in (q, k, v))
    S = Q @ K.T / math.sqrt(32)
    lse_ref = logsumexp(S, axis=1)
    O_ref = np.exp(S - lse_ref[:, None]) @ V
    rows = np.arange(200, dtype=np.int32)
    o, lse = oracle.attention_rows(q, k, v, 0, 0, rows, lib=lib)
    assert np.abs(lse - lse_ref).max() < 1e-11
    assert np.abs(o - O_ref).max() < 1e-11
    # sparse over a key subset equals numpy softmax restricted to that subset
    keys = np.array([3, 17, 18, 99, 150, 199], dtype=np.int32)
    o_s, lse_s = oracle.attention_rows(q, k, v, 0, 0, rows, keys=keys, lib=lib)
    Ss = S[:, keys]
    ls = logsumexp(Ss, axis=1)
    assert np.abs(lse_s - ls).max() < 1e-11
    assert np.abs(o_s - np.exp(Ss - ls[:, None]) @ V[keys]).max() < 1e-11


def check_dense_closed_forms(lib):
    N, d = 64, 16
    rng = np.random.default_rng(2)
    q = _bits(rng.standard_normal((1, N, 1, d)))
    v = _bits(rng.standard_normal((1, N, 1, d)))
    # identical keys: uniform attention, output = mean of V
    k = np.repeat(_bits(rng.standard_normal((1, 1, 1, d))), N, axis=1)
    o, lse = oracle.attention_rows(q, k, v, 0, 0, np.arange(N, dtype=np.int32), lib=lib)
    assert np.abs(o - _wide(v[0, :, 0, :]).mean(axis=0)).max() < 1e-12
    s0 = _wide(q[0, :, 0, :]) @ _wide(k[0, 0, 0, :]) / 4.0
    assert np.abs(lse - (s0 + math.log(N))).max() < 1e-12


def check_mass_sums_to_group_size(lib):
    w, q, k, v = _tiny_qkv(N=300, d=32, seed=4)
    for rows in (np.arange(128, dtype=np.int32), np.array([5, 77, 299], dtype=np.int32)):
        m = oracle.group_mass(q, k, 0, 0, rows, lib=lib)
        assert abs(m.sum() - len(rows)) < 1e-11 and m.min() > 0
        # each row's probabilities sum to one: mass of a single row
        m1 = oracle.group_mass(q, k, 0, 0, rows[:1], lib=lib)
        assert abs(m1.sum() - 1.0) < 1e-13


def test_dense_vs_numpy(orc):
    check_dense_vs_numpy(orc)


def test_dense_closed_forms(orc):
    check_dense_closed_forms(orc)


def test_mass_sums_to_group_size(orc):
    check_mass_sums_to_group_size(orc)


# ---------------------------------------------------------------------------
# top-K
# ---------------------------------------------------------------------------

def check_topk_bruteforce(lib):
    rng = np.random.default_rng(8)
    for N in range(1, 13):
        m = rng.random(N)
        for K in range(0, N + 1):
            got = oracle.topk(m, K, lib=lib)
            best = max(itertools.combinations(range(N), K), key=lambda s: sum(m[list(s)]))
            assert list(got) == list(best), (N, K)


def check_topk_ties_lower_index(lib):
    m = np.array([0.5, 0.2, 0.5, 0.9, 0.2, 0.5, 0.1])
    assert list(oracle.topk(m, 3, lib=lib)) == [0, 2, 3]
    assert list(oracle.topk(m, 5, lib=lib)) == [0, 1, 2, 3, 5]
    assert list(oracle.topk(np.ones(10), 4, lib=lib)) == [0, 1, 2, 3]
    assert list(oracle.topk(m, 7, lib=lib)) == list(range(7))


def test_topk_bruteforce(orc):
    check_topk_bruteforce(orc)


def test_topk_ties_lower_index(orc):
    check_topk_ties_lower_index(orc)


# ---------------------------------------------------------------------------
# anchor sparse pass, residual and reuse
# ---------------------------------------------------------------------------

def check_full_density_zero_residual(lib):
    w, q, k, v = _tiny_qkv(N=256, d=32, seed=12)
    rows = np.arange(0, 256, 2, dtype=np.int32)
    r = oracle.anchor_group(q, k, v, 0, 0, rows, 256, lib=lib)
    assert np.array_equal(r["idx"], np.arange(256))
    assert np.all(r["resid"] == 0.0)


def check_k1_selects_value_row(lib):
    w, q, k, v = _tiny_qkv(N=256, d=32, seed=13)
    rows = np.arange(128, dtype=np.int32)
    r = oracle.anchor_group(q, k, v, 0, 0, rows, 1, lib=lib)
    j = int(r["idx"][0])
    assert j == int(np.argmax(r["mass"]))
    assert np.array_equal(r["o_sparse"], np.repeat(_wide(v[0, j:j + 1, 0, :]), 128, axis=0))


def check_anchor_identity_and_zero_drift_reuse(lib):
    w, q, k, v = _tiny_qkv(N=384, d=32, seed=14)
    rows = np.arange(128, 256, dtype=np.int32)
    r = oracle.anchor_group(q, k, v, 0, 0, rows, 96, lib=lib)
    assert np.abs(r["o_sparse"] + r["resid"] - r["o_dense"]).max() < 1e-14
    # numpy restatement of the anchor's pieces on the selected keys
    Q, K, V = (_wide(t[0, :, 0, :]) for t in (q, k, v))
    S = Q[rows] @ K.T / math.sqrt(32)
    P = np.exp(S - S.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    assert np.abs(r["mass"] - P.sum(axis=0)).max() < 1e-12
    want = np.sort(np.argsort(-P.sum(axis=0), kind="stable")[:96])
    assert np.array_equal(r["idx"], want)
    Ps = np.exp(S[:, want] - S[:, want].max(axis=1, keepdims=True))
    Ps /= Ps.sum(axis=1, keepdims=True)
    assert np.abs(r["o_sparse"] - Ps @ V[want]).max() < 1e-12
    # reuse with unchanged Q/K/V reproduces the dense output
    o = oracle.reuse_group(q, k, v, 0, 0, rows, r["idx"], r["resid"], lib=lib)
    assert np.abs(o - r["o_dense"]).max() < 1e-13


def test_full_density_zero_residual(orc):
    check_full_density_zero_residual(orc)


def test_k1_selects_value_row(orc):
    check_k1_selects_value_row(orc)


def test_anchor_identity_and_zero_drift_reuse(orc):
    check_anchor_identity_and_zero_drift_reuse(orc)


# ---------------------------------------------------------------------------
# metadata format (paper Table 8) and bf16 rounding
# ---------------------------------------------------------------------------

def check_table8_metadata_volume(lib):
    path = os.path.join(ROOT, "tests", "golden", "table8_offload.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 2
    for name, S, H, D, C, Vmb in rows:
        S, H, D, C, Vmb = int(S), int(H), int(D), float(C), float(Vmb)
        K = C * 1e12 / (4 * S * D * H)  # sparse FLOPs C = 4 S K D H
        mb = oracle.metadata_bytes(S, H, D, K, 128)["total"] / 2 ** 20
        assert abs(mb - Vmb) / Vmb < 0.005, (name, mb, Vmb)
        # other plausible formats miss the printed volume by far
        fp32_resid = (S * H * D * 4 + (S / 128) * H * K * 4) / 2 ** 20
        i64_idx = (S * H * D * 2 + (S / 128) * H * K * 8) / 2 ** 20
        assert abs(fp32_resid - Vmb) / Vmb > 0.1 and abs(i64_idx - Vmb) / Vmb > 0.1


def check_round_bf16(lib):
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(5000) * 10.0 ** rng.integers(-6, 6, 5000),
                        [0.0, -0.0, 1.0, -3.5]]).astype(np.float32).astype(np.float64)
    assert np.array_equal(oracle.round_bf16(x, lib=lib), _bits(x))
    # halfway cases resolve to the even neighbour
    one = 1.0
    assert oracle.round_bf16(np.array([one + 2 ** -8]), lib=lib)[0] == 0x3F80
    assert oracle.round_bf16(np.array([one + 3 * 2 ** -8]), lib=lib)[0] == 0x3F82


def check_meta_pack_pins(lib):
    # worked by hand: N = 40, keys {0, 5, 31, 32, 39} -> word 0 has bits 0, 5, 31, word 1 bits 0 and 7
    got = oracle.meta_pack(np.array([[0, 5, 31, 32, 39]]), 40)
    assert got.dtype == np.uint32 and got.tolist() == [[0x80000021, 0x00000081]]
    # every single key of a ragged N lands on its own bit: the row read as one little-endian
    # integer (Python big integers, no numpy bit arithmetic) is 2^j
    N = 77
    for j in range(N):
        w = oracle.meta_pack(np.array([[j]]), N)[0]
        assert sum(int(x) << (32 * i) for i, x in enumerate(w)) == 1 << j
    # random selections: the integer identity, popcount K, nothing at or above N, exact round trip
    rng = np.random.default_rng(7)
    for N, K in [(1000, 333), (777, 1), (64, 64), (4096, 1024)]:
        idx = np.sort(np.stack([rng.choice(N, K, replace=False) for _ in range(5)]), axis=1)
        w = oracle.meta_pack(idx, N)
        assert w.shape == (5, (N + 31) // 32)
        for r in range(5):
            big = sum(int(x) << (32 * i) for i, x in enumerate(w[r]))
            assert big == sum(1 << int(j) for j in idx[r])
            assert big >> N == 0
        assert np.array_equal(oracle.meta_unpack(w, N), idx)
    # K = N: all ones below N
    w = oracle.meta_pack(np.arange(70)[None], 70)[0]
    assert w.tolist() == [0xFFFFFFFF, 0xFFFFFFFF, 0x3F]


def check_krylov_split_pins(lib):
    # SplitMix64 from state 0: the generator's published first outputs
    want = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F, 0xF88BB8A8724C81EC, 0x1B39896A51A8749B]
    assert [oracle.splitmix64(i, lib=lib) for i in range(1, 6)] == want
    rng = np.random.default_rng(11)

    def bf16(x):
        return _bits(np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64))

    # k = 1: the direction is the start vector itself (d = 4, entries from the outputs above)
    d, n = 4, 256
    q = bf16(rng.standard_normal((1, n, 1, d)))
    r = oracle.pddp_split_krylov(q, 0, 0, np.arange(n), 1, lib=lib)
    v0 = np.array([1.0 + (x >> 11) * 2.0 ** -53 for x in want[:d]])
    v0 /= np.linalg.norm(v0)
    v0 *= np.sign(v0[np.argmax(np.abs(v0))])
    assert np.abs(r["dir"] - v0).max() < 1e-15
    # k = d: the Krylov space is the whole space, so the split is the exact method's
    d, n = 16, 300
    scales = np.linspace(3.0, 0.5, d)
    q = bf16(rng.standard_normal((1, n, 1, d)) * scales)
    rk = oracle.pddp_split_krylov(q, 0, 0, np.arange(n), d, lib=lib)
    rx = oracle.pddp_split(q, 0, 0, np.arange(n), lib=lib)
    assert abs(abs(np.dot(rk["dir"], rx["dir"])) - 1.0) < 1e-10
    assert np.array_equal(rk["left"], rx["left"])
    # rank-2 data: three Krylov steps contain C's range, so the direction is the top axis u1
    d, n = 32, 512
    u = np.linalg.qr(rng.standard_normal((d, 2)))[0]
    a, c = 2.0 ** rng.integers(-3, 3, n) * rng.choice([-1, 1], n), rng.choice([-0.25, 0.25], n)
    x = np.outer(a, u[:, 0]) + np.outer(c, u[:, 1])
    q = bf16(x[None, :, None, :])
    xe = _wide(q)[0, :, 0, :]  # the exact bf16 values the oracle sees
    w, V = np.linalg.eigh(np.cov(xe.T, bias=True) * n)
    top = V[:, -1]
    r = oracle.pddp_split_krylov(q, 0, 0, np.arange(n), 3, lib=lib)
    assert abs(abs(np.dot(r["dir"], top)) - 1.0) < 1e-10
    assert w[-1] > 10 * w[-2]


def check_whitening_pins(lib):
    """Whitened grouping = PDDP on the per-channel standardised queries."""
    rng = np.random.default_rng(23)
    # channel scales against numpy's population std; a constant channel keeps scale 1
    n, d = 300, 8
    x = rng.standard_normal((n, d)) * 2.0 ** rng.integers(-3, 4, d)
    x[:, 5] = 0.75
    q = _bits(x[None, :, None, :])
    xe = _wide(q)[0, :, 0, :]
    sd = xe.std(axis=0)
    want = np.where(sd > 0, 1.0 / np.where(sd > 0, sd, 1.0), 1.0)
    got = oracle.channel_scale(q, 0, 0, lib=lib)
    assert np.allclose(got, want, rtol=1e-12, atol=0) and got[5] == 1.0
    # exact invariance: scaling a channel by a power of two (exact in bf16) leaves the whitened
    # queries, and so the whitened grouping, unchanged bit for bit; the plain grouping changes
    n, d = 700, 16
    x = rng.standard_normal((n, d)) * np.linspace(2.0, 0.5, d)
    k = np.array([6, -2, 0, 3, 1, -3, 2, 0, 4, -1, 0, 2, -2, 1, 0, 3])
    q1 = _bits(x[None, :, None, :])
    q2 = _bits((_wide(q1)[0, :, 0, :] * 2.0 ** k)[None, :, None, :])
    assert np.array_equal(_wide(q2)[0, :, 0, :], _wide(q1)[0, :, 0, :] * 2.0 ** k)
    p1, p2 = oracle.pddp_whitened(q1, 0, 0, lib=lib), oracle.pddp_whitened(q2, 0, 0, lib=lib)
    assert np.array_equal(p1, p2)
    assert not np.array_equal(oracle.pddp(q1, 0, 0, lib=lib)[0], oracle.pddp(q2, 0, 0, lib=lib)[0])
    # one channel of large independent variance and seven channels sharing a latent: the plain
    # direction is that channel, the whitened direction the shared latent's (1, ..., 1) / sqrt(7)
    n = 512
    u = rng.integers(-8, 9, n) * 64.0
    v = rng.integers(-8, 9, n).astype(np.float64)
    x = np.concatenate([u[:, None], v[:, None] + rng.choice([-0.5, 0.0, 0.5], (n, 7))], axis=1)
    q = _bits(x[None, :, None, :])
    assert np.array_equal(_wide(q)[0, :, 0, :], x)
    plain = oracle.pddp_split(q, 0, 0, np.arange(n), lib=lib)
    white = oracle.pddp_split(q, 0, 0, np.arange(n), lib=lib, wscale=oracle.channel_scale(q, 0, 0, lib=lib))
    assert abs(plain["dir"][0]) > 0.999
    assert abs(white["dir"][0]) < 0.1 and np.abs(white["dir"][1:] - 7 ** -0.5).max() < 0.05


def test_krylov_split_pins(orc):
    check_krylov_split_pins(orc)


def test_whitening_pins(orc):
    check_whitening_pins(orc)


def test_meta_pack_pins(orc):
    check_meta_pack_pins(orc)


def test_table8_metadata_volume(orc):
    check_table8_metadata_volume(orc)


def test_round_bf16(orc):
    check_round_bf16(orc)


ALL_CHECKS = [
    check_jacobi_vs_numpy, check_jacobi_2x2_closed_form, check_pddp_rank1_sorts_by_latent,
    check_pddp_matches_numpy_projection, check_pddp_sizes_and_leaves, check_dense_vs_numpy,
    check_dense_closed_forms, check_mass_sums_to_group_size, check_topk_bruteforce, check_topk_ties_lower_index,
    check_full_density_zero_residual, check_k1_selects_value_row, check_anchor_identity_and_zero_drift_reuse,
    check_round_bf16, check_meta_pack_pins, check_krylov_split_pins, check_whitening_pins,
]
