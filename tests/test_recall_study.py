"""Selection granularity and query grouping on synthetic data (the paper's Table 4, reproduced in kind).

For a smooth 3-D synthetic field (4 x 32 x 32 tokens, d = 64) and densities
s = 0.1, 0.2, 0.3, the fp64 oracle measures, per configuration:
  attention recall  mean over queries of the exact probability mass on the
                    selected keys (a group's selected mass over its size, since
                    each query's probabilities sum to 1);
  output rel. L1    sum |O_sparse - O_dense| / sum |O_dense| (renormalised
                    sparse attention, no residual);
for groupings {token order, PDDP} x KV granularity {token, 64-key blocks}, at
matched density (K = s*N rounded to whole blocks, the same K for both).
Checked: token selection never recalls less than block selection (top-K of the
group mass maximises the selected mass over all K-key sets), and on this field
PDDP grouping raises token-granular recall and lowers the output error at every
density. The table is printed (pytest -s) for the design notes.
"""
import numpy as np
import pytest

import oracle
import synth

DENSITIES = (0.1, 0.2, 0.3)
BLOCK = 64


def _study(w, threads=16):
    q, k, v = (synth.generate(w, t) for t in "qkv")
    N = w.N
    G = (N + 127) // 128
    out = {}
    for grouping in ("token order", "pddp"):
        perm = np.arange(N, dtype=np.int32) if grouping == "token order" else oracle.pddp(q, 0, 0)[0]
        for s in DENSITIES:
            K = int(round(s * N / BLOCK)) * BLOCK
            nb = K // BLOCK

            def one(g):
                rows = perm[g * 128:(g + 1) * 128]
                a = oracle.anchor_group(q, k, v, 0, 0, rows, K)
                od = a["o_dense"]
                bmass = np.add.reduceat(a["mass"], np.arange(0, N, BLOCK))
                top = np.lexsort((np.arange(len(bmass)), -bmass))[:nb]  # largest block mass, lower block on ties
                keys = np.sort(np.concatenate([np.arange(b * BLOCK, min(N, (b + 1) * BLOCK)) for b in top]))
                ob, _ = oracle.attention_rows(q, k, v, 0, 0, rows, keys=keys.astype(np.int32))
                return (a["mass"][a["idx"]].sum(), a["mass"][keys].sum(), np.abs(a["o_sparse"] - od).sum(),
                        np.abs(ob - od).sum(), np.abs(od).sum(), len(rows))

            t = np.array(oracle.run_groups(one, range(G), threads)).sum(0)
            out[(grouping, s)] = dict(recall_token=t[0] / t[5], recall_block=t[1] / t[5],
                                      rel_l1_token=t[2] / t[4], rel_l1_block=t[3] / t[4])
    return out


@pytest.fixture(scope="module")
def table():
    w = synth.Workload("recall_study", H=1, N=4096, d=64, density=0.2, grid=(4, 32, 32), model=1, seed=1101)
    return _study(w)


def test_print_table(table):
    print("\ngrouping     s    recall(token) recall(block) relL1(token) relL1(block)")
    for (g, s), r in table.items():
        print(f"{g:12s} {s:.1f}  {r['recall_token']:.3f}         {r['recall_block']:.3f}         "
              f"{r['rel_l1_token']:.3f}        {r['rel_l1_block']:.3f}")


def test_token_selection_recalls_at_least_block_selection(table):
    for key, r in table.items():
        assert r["recall_token"] >= r["recall_block"] - 1e-12, key


def test_grouping_helps_token_granular_selection(table):
    for s in DENSITIES:
        ident, pddp = table[("token order", s)], table[("pddp", s)]
        assert pddp["recall_token"] > ident["recall_token"], s
        assert pddp["rel_l1_token"] < ident["rel_l1_token"], s


def test_recall_grows_with_density(table):
    for g in ("token order", "pddp"):
        rec = [table[(g, s)]["recall_token"] for s in DENSITIES]
        assert rec[0] < rec[1] < rec[2] <= 1.0
