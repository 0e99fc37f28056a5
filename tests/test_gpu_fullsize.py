"""Full-size workloads in the benchmark's launch configuration, checked on
samples the oracle can compute one by one.

- Grouping and the anchor on it: for sampled groups g, the oracle walks its
  own PDDP tree from all N queries down to leaf g (its own member sets, never
  the GPU's). At every node on the way the GPU's left child must hold the
  same queries (near ties below 1e-6 relative excepted; a walk that meets one
  stops there). At the leaf the oracle's member set is the GPU's group g, and
  the oracle's anchor on those queries is compared with the GPU anchor run on
  the GPU's own grouping: KV indices exact except near ties, the anchor output
  O, the residual R and the lse, then the reuse step.
- A second anchor and reuse run with a seeded test-made permutation (queries
  with no spatial coherence, so much flatter group masses) is checked the same
  way on sampled groups.
- The lse: relative error at most 1e-6 against the oracle on every compared
  row (the precision the fp64 selection re-score divides by). The softmax side
  of the dense pass contributes a few 1e-7 at most (fp64 row sums, an exact
  exponent, MUFU ex2 rounding); the rest is the tensor core's fp32
  accumulation of the scores themselves, a few ulp of the largest scores of a
  row (largest with the heavy-tailed keys of the MiniMax-H3-shaped case).
"""
import os

import numpy as np
import pytest

import oracle
import synth
from helpers import assert_close, f64, from_dev_bf16, index_mismatches_ok, to_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

THREADS = max(1, min(32, os.cpu_count() or 1))
LSE_REL = 1e-6

# workload name, density (None: the workload's own)
CASES = [("wan13b_480p", None), ("wan14b_720p", None), ("h3_768p", None), ("h3_768p", 0.25), ("asset3d", None)]


@pytest.fixture(scope="module")
def mcs():
    import free_sparse_attention_pddp_b200 as m

    m.load()
    return m


def oracle_walk(q_head, perm_gpu, g, rel=1e-6):
    """The oracle's member set of leaf g (ascending), reached by its own splits
    from the root; at every node the GPU's left child must match. Returns None
    when a near tie (|p - p_split| <= rel * max|p|) makes the trees diverge."""
    N = perm_gpu.shape[0]
    off, mem = 0, np.arange(N, dtype=np.int32)
    lo = g * 128
    while (len(mem) + 127) // 128 > 1:
        r = oracle.pddp_split(q_head, 0, 0, mem, 128)
        L = len(r["left"])
        diff = set(map(int, perm_gpu[off:off + L])) ^ set(map(int, r["left"]))
        if diff:
            proj = dict(zip(map(int, mem), r["proj"]))
            pmax = np.abs(r["proj"]).max()
            assert all(abs(proj[j] - r["split_p"]) <= rel * pmax for j in diff), (off, len(mem))
            return None
        if lo < off + L:
            mem = r["left"]
        else:
            off, mem = off + L, r["right"]
    assert off == lo
    return np.sort(mem).astype(np.int32)


def run_path(mcs, shape, q, k, v, q1, k1, v1, perm):
    B, H, N, d, K = shape.B, shape.H, shape.N, shape.d, shape.topk
    G = (N + 127) // 128
    idx = torch.empty(B, H, G, K, dtype=torch.int32, device="cuda")
    resid = torch.empty(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
    o0 = torch.empty_like(q)
    o1 = torch.empty_like(q)
    wsa = mcs.workspace(shape, mcs.MCS_OP_ANCHOR)
    mcs.mcs_anchor(shape, q, k, v, perm, o0, idx, resid, lse, wsa)
    st, info = mcs.mcs_poll_status(wsa)
    assert st == 0 and info[2] == 0, info
    del wsa
    wss = mcs.workspace(shape, mcs.MCS_OP_SPARSE)
    mcs.mcs_sparse(shape, q1, k1, v1, perm, idx, resid, o1, wss)
    assert mcs.mcs_poll_status(wss)[0] == 0
    # bf16 bit patterns; compared rows are widened one group at a time
    return dict(idx=idx.cpu().numpy(), resid=from_dev_bf16(resid), lse=lse.cpu().numpy().astype(np.float64),
                o0=from_dev_bf16(o0), o1=from_dev_bf16(o1))


def compare_group(name, tag, out, h, g, rows, tok_pos, a, o_ref, K):
    """GPU results of group g (head h) against the oracle's anchor `a` on `rows`.
    tok_pos maps a token to its row in the GPU's permutation order."""
    n_mis, n_bad = index_mismatches_ok(out["idx"][0, h, g], a["idx"], a["mass"], K)
    assert n_bad == 0, (name, tag, h, g, n_mis)
    assert_close(f64(out["o0"][0, rows, h]), a["o_dense"], f"{name} {tag} anchor o h{h} g{g}")
    r_gpu = f64(out["resid"][0, h, [tok_pos[int(t)] for t in rows]])
    assert_close(r_gpu, a["resid"], f"{name} {tag} resid h{h} g{g}")
    lse_gpu = out["lse"][0, h, rows]
    rel = np.abs(lse_gpu - a["lse"]) / np.abs(a["lse"])
    assert rel.max() <= LSE_REL, (name, tag, h, g, float(rel.max()), float(np.abs(lse_gpu - a["lse"]).max()))
    if n_mis == 0:
        assert_close(f64(out["o1"][0, rows, h]), o_ref, f"{name} {tag} reuse o h{h} g{g}")
    return float(np.abs(lse_gpu - a["lse"]).max()), float(rel.max()), n_mis


@pytest.mark.parametrize("name,density", CASES, ids=[f"{n}-{d or 'base'}" for n, d in CASES])
def test_fullsize_sampled(mcs, name, density):
    w = synth.WORKLOADS[name]
    B, H, N, d, G = w.B, w.H, w.N, w.d, w.G
    K = w.topk if density is None else synth.topk_for(N, density)
    sample_heads = [0, H - 1]
    host = {(t, s): synth.generate(w, t, s) for t in "qkv" for s in (0, 1)}
    dq0, dk0, dv0, dq1, dk1, dv1 = (to_dev(host[(t, s)]) for s in (0, 1) for t in "qkv")
    shape = mcs.Shape(B, H, N, d, topk=K)
    # grouping on the full tensor
    perm = torch.empty(B, H, N, dtype=torch.int32, device="cuda")
    wsg = mcs.workspace(shape, mcs.MCS_OP_GROUP)
    mcs.mcs_group(shape, dq0, perm, wsg)
    assert mcs.mcs_poll_status(wsg)[0] == 0
    del wsg
    P = perm.cpu().numpy()
    for h in range(H):
        assert np.array_equal(np.sort(P[0, h]), np.arange(N))
    gpu_grp = run_path(mcs, shape, dq0, dk0, dv0, dq1, dk1, dv1, perm)
    # a seeded test-made permutation: flat, incoherent groups
    tperm = np.stack([np.random.default_rng(100 + h).permutation(N).astype(np.int32) for h in range(H)])[None]
    test_grp = run_path(mcs, shape, dq0, dk0, dv0, dq1, dk1, dv1, torch.from_numpy(tperm).cuda())
    del dq0, dk0, dv0, dq1, dk1, dv1, perm

    rng = np.random.default_rng(7)
    groups = [0, G - 1] + sorted(rng.choice(np.arange(1, G - 1), size=2, replace=False).tolist())
    q_heads = {h: np.ascontiguousarray(host[("q", 0)][:, :, h:h + 1, :]) for h in sample_heads}

    def one(job):
        kind, h, g = job
        if kind == "pddp":
            rows = oracle_walk(q_heads[h], P[0, h], g)
            if rows is None:
                return job, None, None, None
        else:
            rows = tperm[0, h, g * 128:(g + 1) * 128]
        a = oracle.anchor_group(host[("q", 0)], host[("k", 0)], host[("v", 0)], 0, h, rows, K)
        o_ref = oracle.reuse_group(host[("q", 1)], host[("k", 1)], host[("v", 1)], 0, h, rows, a["idx"], a["resid"])
        return job, rows, a, o_ref

    jobs = [(kind, h, g) for kind in ("pddp", "test") for h in sample_heads for g in groups]
    pos = {("pddp", h): np.argsort(P[0, h]) for h in sample_heads}
    pos.update({("test", h): np.argsort(tperm[0, h]) for h in sample_heads})
    walked = lse_max = lse_rel = 0
    for (kind, h, g), rows, a, o_ref in oracle.run_groups(one, jobs, THREADS):
        if rows is None:
            continue
        out = gpu_grp if kind == "pddp" else test_grp
        if kind == "pddp":
            walked += 1
            # the oracle's leaf is the GPU's group g
            assert np.array_equal(np.sort(P[0, h, g * 128:(g + 1) * 128]), rows), (name, h, g)
        err, rel, _ = compare_group(name, kind, out, h, g, rows, pos[(kind, h)], a, o_ref, K)
        lse_max, lse_rel = max(lse_max, err), max(lse_rel, rel)
    assert walked >= len(groups), (name, walked)  # most walks reach their leaf
    print(f"{name} K={K}: {walked} groups on the GPU grouping, max |lse - oracle| {lse_max:.3e} "
          f"(relative {lse_rel:.3e})")
