"""Shared test helpers: device upload of synthetic inputs and the output tolerances.

Tolerances (bf16 inputs, fp32 accumulation, bf16 outputs): max-abs 2e-2 and
mean-abs 2e-3 against the fp64 oracle.
"""
import numpy as np

import oracle
import synth

MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def to_dev(bits: np.ndarray):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def from_dev_bf16(t) -> np.ndarray:
    import torch

    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f64(bits):
    return synth.bf16_to_f64(bits)


def assert_close(got, want, what, max_abs=MAX_ABS, mean_abs=MEAN_ABS):
    err = np.abs(np.asarray(got, dtype=np.float64) - np.asarray(want, dtype=np.float64))
    assert err.max() <= max_abs and err.mean() <= mean_abs, (
        f"{what}: max-abs {err.max():.3e} (<= {max_abs}), mean-abs {err.mean():.3e} (<= {mean_abs})")
    return err.max(), err.mean()


def oracle_metadata(q, k, v, K, heads=None, threads=8, perm=None):
    """Oracle anchor for every group: perm [B,H,N], kv_idx [B,H,G,K], resid fp64 [B,H,N,d] (perm order),
    o_dense fp64 [B,H,N,d] (perm order), lse [B,H,N] (perm order)."""
    B, N, H, d = q.shape
    G = (N + 127) // 128
    heads = range(H) if heads is None else heads
    P = np.zeros((B, H, N), np.int32)
    IDX = np.zeros((B, H, G, K), np.int32)
    R = np.zeros((B, H, N, d))
    OD = np.zeros((B, H, N, d))
    LSE = np.zeros((B, H, N))
    for b in range(B):
        for h in heads:
            P[b, h] = perm[b, h] if perm is not None else oracle.pddp(q, b, h)[0]

            def one(g):
                rows = P[b, h, g * 128:(g + 1) * 128]
                return g, oracle.anchor_group(q, k, v, b, h, rows, K)

            for g, r in oracle.run_groups(one, range(G), threads):
                IDX[b, h, g] = r["idx"]
                R[b, h, g * 128:g * 128 + len(r["lse"])] = r["resid"]
                OD[b, h, g * 128:g * 128 + len(r["lse"])] = r["o_dense"]
                LSE[b, h, g * 128:g * 128 + len(r["lse"])] = r["lse"]
    return P, IDX, R, OD, LSE


def index_mismatches_ok(got_idx, want_idx, mass, K, rel=1e-6):
    """Compare one group's KV index list with the oracle's.

    Returns (n_mismatch, n_unexplained): a mismatching index is explained when
    its oracle mass lies within rel * m_(K) of the K-th largest oracle mass
    m_(K) (a near tie at the selection boundary).
    """
    got, want = set(map(int, got_idx)), set(map(int, want_idx))
    diff = got ^ want
    if not diff:
        return 0, 0
    mK = np.sort(mass)[::-1][K - 1]
    bad = [j for j in diff if abs(mass[j] - mK) > rel * mK]
    return len(diff), len(bad)


def check_kv_idx_valid(idx, N, K):
    """kv_idx rows: exactly K strictly ascending indices in [0, N)."""
    idx = np.asarray(idx)
    assert idx.shape[-1] == K
    assert idx.min() >= 0 and idx.max() < N
    assert np.all(np.diff(idx, axis=-1) > 0)


def pddp_replay(q, b, h, perm, g=128, rel=1e-6, gap_min=1e-4, wscale=None):
    """Check a grouping node by node against the oracle's split of the same member set
    (``wscale``: the whitened grouping's channel scales, from oracle.channel_scale).

    For every internal node of the tree (its shape depends only on N), the
    oracle splits the GPU's member set; the GPU's left child must equal the
    oracle's, except for members whose oracle projection is within
    rel * max|p| of the split value, or at nodes whose relative eigengap is
    below gap_min (reported). Returns (nodes, exact_nodes, tolerated, weak_gap_nodes).
    """
    N = perm.shape[0]
    nodes = oracle.pddp_tree(N, g)
    exact = tolerated = weak = 0
    for off, n, L in nodes:
        mem = np.sort(perm[off:off + n])
        r = oracle.pddp_split(q, b, h, mem, g, wscale=wscale)
        gap = (r["eig"][0] - r["eig"][1]) / r["eig"][0]
        got_left = set(map(int, perm[off:off + L]))
        want_left = set(map(int, r["left"]))
        diff = got_left ^ want_left
        if not diff:
            exact += 1
            continue
        if gap < gap_min:
            weak += 1
            continue
        proj = dict(zip(map(int, mem), r["proj"]))
        pmax = np.abs(r["proj"]).max()
        for j in diff:
            assert abs(proj[j] - r["split_p"]) <= rel * pmax, (
                f"node off={off} n={n}: token {j} split differently, |p - p_split| = "
                f"{abs(proj[j] - r['split_p']):.3e} > {rel} * {pmax:.3e}")
        tolerated += 1
    return len(nodes), exact, tolerated, weak
