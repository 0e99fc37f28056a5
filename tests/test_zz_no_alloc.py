"""The workspace-free reuse step (mcs_sparse_noalloc) against the regular one.

Callers that cannot allocate device memory where they run the reuse step (a
runtime that reserves all device memory up front and hands out only tensor
buffers, or a plug-in that must not touch the allocator) use this entry point;
its status block lives in a static device array instead of a workspace. Both
entry points launch the same kernel on the same inputs, so their outputs must
agree bit for bit. This file is collected last so that, if it fails, a run
stopping at the first failure has already run every other test; it also
passes on its own in a fresh process.
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import to_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def test_noalloc_reuse_matches_workspace_reuse_twice():
    import free_sparse_attention_pddp_b200 as mcs

    N, H, d, K = 1000, 2, 128, 333
    w = synth.small(N, H=H, d=d, seed=61)
    q, k, v = (to_dev(synth.generate(w, t, 1)) for t in "qkv")
    G = (N + 127) // 128
    rng = np.random.default_rng(3)
    perm = np.stack([rng.permutation(N).astype(np.int32) for _ in range(H)])[None]
    idx = np.sort(np.stack([[rng.choice(N, K, replace=False) for _ in range(G)] for _ in range(H)]), axis=-1)
    idx = idx.astype(np.int32)[None]
    resid = oracle.round_bf16(rng.standard_normal((1, H, N, d)) * 0.05)
    dP, dI = torch.from_numpy(perm).cuda(), torch.from_numpy(idx).cuda()
    dR = torch.from_numpy(resid.view(np.int16)).view(torch.bfloat16).cuda()
    shape = mcs.Shape(1, H, N, d, topk=K)
    ref = torch.empty(1, N, H, d, dtype=torch.bfloat16, device="cuda")
    ws = mcs.workspace(shape, mcs.MCS_OP_SPARSE)
    mcs.mcs_sparse(shape, q, k, v, dP, dI, dR, ref, ws)
    assert mcs.mcs_poll_status(ws)[0] == 0
    for call in range(2):  # the static scratch keeps the previous call's contents
        out = torch.full_like(ref, float("nan"))
        info = mcs.mcs_sparse_noalloc(shape, q, k, v, dP, dI, dR, out)
        assert info[0] == 0, info
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"no-alloc reuse, call {call}"
    # a device-side error reaches the caller through the static status block ...
    bad = dI.clone()
    bad[0, 1, 3, 7] = N  # out of range
    with pytest.raises(mcs.MCSError) as e:
        mcs.mcs_sparse_noalloc(shape, q, k, v, dP, bad, dR, torch.empty_like(ref))
    assert e.value.code == 5  # MCS_ERR_BAD_INDEX
    # ... and the next clean call starts from a cleared block
    out = torch.empty_like(ref)
    info = mcs.mcs_sparse_noalloc(shape, q, k, v, dP, dI, dR, out)
    assert info[0] == 0 and info[1] == 0, info
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_noalloc_rejects_bad_arguments():
    import free_sparse_attention_pddp_b200 as mcs

    shape = mcs.Shape(1, 1, 256, 96, topk=8)  # d = 96 is unsupported
    x = torch.zeros(1, 256, 1, 96, dtype=torch.bfloat16, device="cuda")
    i = torch.zeros(1, 1, 2, 8, dtype=torch.int32, device="cuda")
    p = torch.zeros(1, 1, 256, dtype=torch.int32, device="cuda")
    with pytest.raises(mcs.MCSError) as e:
        mcs.mcs_sparse_noalloc(shape, x, x, x, p, i, None, x)
    assert e.value.code == 2
