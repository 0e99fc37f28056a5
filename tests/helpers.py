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
