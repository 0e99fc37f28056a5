"""GPU: the host-buffer reuse step (mcs_sparse_host) against mcs_sparse.

mcs_sparse_host splits the heads into chunks and chains, per chunk, the copy of
its q/k/v columns in, the reuse kernel over those heads and the copy of its o
columns out, on three streams. Its arithmetic is mcs_sparse's, so the output
must be bit-identical for every chunk count (one chunk, several, one per head,
counts that do not divide H). mcs_sparse itself is checked against the oracle
elsewhere; the metadata here only has to be valid (a permutation per head,
ascending distinct key indices per group, a finite residual).
"""
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mcs():
    import free_sparse_attention_pddp_b200 as m

    m.load()
    return m


def _case(B, H, N, d, K, seed):
    g = torch.Generator().manual_seed(seed)
    qkv = [torch.randn(B, N, H, d, generator=g).to(torch.bfloat16) for _ in range(3)]
    G = (N + 127) // 128
    perm = torch.stack([torch.stack([torch.randperm(N, generator=g) for _ in range(H)]) for _ in range(B)])
    idx = torch.empty(B, H, G, K, dtype=torch.int32)
    for b in range(B):
        for h in range(H):
            for t in range(G):
                idx[b, h, t] = torch.randperm(N, generator=g)[:K].sort().values
    resid = (0.1 * torch.randn(B, H, N, d, generator=g)).to(torch.bfloat16)
    return qkv, perm.to(torch.int32), idx, resid


def _run_both(mcs, B, H, N, d, K, seed, chunks, with_resid=True):
    (q, k, v), perm, idx, resid = _case(B, H, N, d, K, seed)
    shape = mcs.Shape(B, H, N, d, topk=K)
    dP, dI = perm.cuda(), idx.cuda()
    dR = resid.cuda() if with_resid else None
    ws = mcs.workspace(shape, mcs.MCS_OP_SPARSE)
    o_ref = torch.empty(B, N, H, d, dtype=torch.bfloat16, device="cuda")
    mcs.mcs_sparse(shape, q.cuda(), k.cuda(), v.cuda(), dP, dI, dR, o_ref, ws)
    st, info = mcs.mcs_poll_status(ws)
    assert st == 0, info
    host = [t.pin_memory() for t in (q, k, v)]
    dev = [torch.empty_like(t, device="cuda") for t in (q, k, v)]
    main = torch.cuda.Stream()
    cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    for c in chunks:
        o_host = torch.full((B, N, H, d), float("nan"), dtype=torch.bfloat16).pin_memory()
        o_dev = torch.full((B, N, H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
        torch.cuda.synchronize()
        mcs.mcs_sparse_host(shape, *host, dP, dI, dR, o_host, *dev, o_dev, c, ws, main, cin, cout)
        main.synchronize()  # the call orders `main` after its last output copy
        st, info = mcs.mcs_poll_status(ws, main)
        assert st == 0, (c, info)
        outs.append((c, o_host.clone(), o_dev.cpu()))
    return o_ref.cpu(), outs


@pytest.mark.parametrize("B,H,N,d,K,seed", [
    (2, 5, 700, 128, 200, 71),   # ragged N and K tails, odd head count
    (1, 6, 1000, 64, 333, 72),
])
def test_host_pipeline_bit_identical(mcs, B, H, N, d, K, seed):
    chunks = sorted({1, 2, 3, H})
    o_ref, outs = _run_both(mcs, B, H, N, d, K, seed, chunks)
    for c, o_host, o_dev in outs:
        assert torch.equal(o_host.view(torch.int16), o_ref.view(torch.int16)), f"head_chunks={c}: host output"
        assert torch.equal(o_dev.view(torch.int16), o_ref.view(torch.int16)), f"head_chunks={c}: device output"


def test_host_pipeline_without_residual(mcs):
    o_ref, outs = _run_both(mcs, 1, 4, 513, 128, 130, 73, [3], with_resid=False)
    assert torch.equal(outs[0][1].view(torch.int16), o_ref.view(torch.int16))


def test_host_pipeline_argument_errors(mcs):
    B, H, N, d, K = 1, 3, 256, 128, 64
    (q, k, v), perm, idx, resid = _case(B, H, N, d, K, 74)
    shape = mcs.Shape(B, H, N, d, topk=K)
    ws = mcs.workspace(shape, mcs.MCS_OP_SPARSE)
    host = [t.pin_memory() for t in (q, k, v)]
    dev = [torch.empty_like(t, device="cuda") for t in (q, k, v)]
    o_host = torch.empty(B, N, H, d, dtype=torch.bfloat16).pin_memory()
    o_dev = torch.empty(B, N, H, d, dtype=torch.bfloat16, device="cuda")
    s = [torch.cuda.Stream() for _ in range(3)]
    for chunks in (0, -1, H + 1):
        with pytest.raises(mcs.MCSError):
            mcs.mcs_sparse_host(shape, *host, perm.cuda(), idx.cuda(), None, o_host, *dev, o_dev, chunks, ws, *s)
    with pytest.raises(mcs.MCSError):  # missing device buffer
        mcs.mcs_sparse_host(shape, *host, perm.cuda(), idx.cuda(), None, o_host, dev[0], dev[1], None, o_dev, 1, ws,
                            *s)
    with pytest.raises(mcs.MCSError):  # missing host buffer
        mcs.mcs_sparse_host(shape, host[0], None, host[2], perm.cuda(), idx.cuda(), None, o_host, *dev, o_dev, 1,
                            ws, *s)
