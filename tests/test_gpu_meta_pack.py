"""GPU parity of the packed selection (mcs_meta_pack / mcs_meta_unpack) against the oracle.

Packing is bit-exact integer work: the device mask must equal the oracle's word
for word, and unpacking must give back the ascending lists exactly. Cases span
ragged N (not a multiple of 32), K = 1, K = N, several rows, and the offload
workload's full size; malformed inputs must raise MCS_ERR_BAD_INDEX in the status
block without writing outside the destination.
"""
import numpy as np
import pytest

import oracle

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mcs():
    import free_sparse_attention_pddp_b200 as m

    m.load()
    return m


def _lists(B, H, N, K, seed):
    rng = np.random.default_rng(seed)
    G = (N + 127) // 128
    idx = np.empty((B, H, G, K), np.int32)
    for r in np.ndindex(B, H, G):
        idx[r] = np.sort(rng.choice(N, K, replace=False))
    return idx


def _roundtrip(mcs, B, H, N, K, idx):
    shape = mcs.Shape(B, H, N, 64, topk=K)
    G = (N + 127) // 128
    W = (N + 31) // 32
    assert mcs.mcs_meta_mask_bytes(shape) == B * H * G * W * 4
    ws = mcs.workspace(shape, mcs.MCS_OP_SPARSE)
    d_idx = torch.from_numpy(idx).cuda()
    mask = torch.full((B, H, G, W), -1, dtype=torch.int32, device="cuda")
    mcs.mcs_meta_pack(shape, d_idx, mask, ws)
    back = torch.full_like(d_idx, -7)
    mcs.mcs_meta_unpack(shape, mask, back, ws)
    st, info = mcs.mcs_poll_status(ws)
    assert st == 0, info
    return mask.cpu().numpy().view(np.uint32), back.cpu().numpy()


@pytest.mark.parametrize("B,H,N,K,seed", [
    (1, 2, 1000, 333, 81),   # ragged N, several groups
    (2, 1, 777, 1, 82),      # K = 1
    (1, 1, 300, 300, 83),    # K = N: every key
    (1, 3, 4096, 819, 84),   # N a multiple of 32
    (1, 1, 33, 17, 85),      # one full word and one bit of the next
])
def test_pack_unpack_match_oracle(mcs, B, H, N, K, seed):
    idx = _lists(B, H, N, K, seed)
    mask, back = _roundtrip(mcs, B, H, N, K, idx)
    assert np.array_equal(mask, oracle.meta_pack(idx, N))
    assert np.array_equal(back, idx)


def test_pack_unpack_offload_size(mcs):
    """The offload workload's shape (16 heads, N = 65536, K = 9830): sampled rows against the oracle."""
    B, H, N, K = 1, 16, 65536, 9830
    G = (N + 127) // 128
    shape = mcs.Shape(B, H, N, 64, topk=K)
    ws = mcs.workspace(shape, mcs.MCS_OP_SPARSE)
    g = torch.Generator(device="cuda").manual_seed(86)
    # ascending distinct lists: the tokens of the K largest of a random score, sorted
    keys = torch.rand(B * H * G, N, generator=g, device="cuda")
    d_idx = keys.topk(K, dim=1).indices.sort(dim=1).values.to(torch.int32).view(B, H, G, K)
    del keys
    mask = torch.empty(mcs.mcs_meta_mask_bytes(shape) // 4, dtype=torch.int32, device="cuda")
    mcs.mcs_meta_pack(shape, d_idx, mask, ws)
    back = torch.empty_like(d_idx)
    mcs.mcs_meta_unpack(shape, mask, back, ws)
    st, info = mcs.mcs_poll_status(ws)
    assert st == 0, info
    assert torch.equal(back, d_idx)
    rows = np.random.default_rng(86).choice(B * H * G, 24, replace=False)
    W = (N + 31) // 32
    m = mask.view(B * H * G, W)[torch.from_numpy(rows).cuda()].cpu().numpy().view(np.uint32)
    want = oracle.meta_pack(d_idx.view(B * H * G, K)[torch.from_numpy(rows).cuda()].cpu().numpy(), N)
    assert np.array_equal(m, want)


def test_pack_through_host_and_back(mcs):
    """Offload round trip: pack, copy to pinned host memory and back with mcs_meta_copy, unpack."""
    B, H, N, K = 1, 2, 2000, 400
    idx = _lists(B, H, N, K, 87)
    shape = mcs.Shape(B, H, N, 128, topk=K)
    ws = mcs.workspace(shape, mcs.MCS_OP_SPARSE)
    nbytes = mcs.mcs_meta_mask_bytes(shape)
    mask = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    mcs.mcs_meta_pack(shape, torch.from_numpy(idx).cuda(), mask, ws)
    host = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    side = torch.cuda.Stream()
    done = torch.cuda.Event()
    packed = torch.cuda.Event()
    packed.record()
    mcs.mcs_meta_copy(host, mask, nbytes, True, side, wait_event=packed, done_event=done)
    done.synchronize()
    mask2 = torch.zeros_like(mask)
    side.wait_stream(torch.cuda.current_stream())  # the zero fill lands before the copy back
    mcs.mcs_meta_copy(mask2, host, nbytes, False, side, done_event=done)
    torch.cuda.current_stream().wait_event(done)
    back = torch.empty(B, H, (N + 127) // 128, K, dtype=torch.int32, device="cuda")
    mcs.mcs_meta_unpack(shape, mask2, back, ws)
    st, info = mcs.mcs_poll_status(ws)
    assert st == 0, info
    assert np.array_equal(back.cpu().numpy(), idx)
    assert np.array_equal(host.numpy().view(np.uint32).reshape(B, H, -1, (N + 31) // 32), oracle.meta_pack(idx, N))


def test_malformed_inputs_report_bad_index(mcs):
    B, H, N, K = 1, 1, 500, 50
    shape = mcs.Shape(B, H, N, 64, topk=K)
    G = (N + 127) // 128
    W = (N + 31) // 32
    ws = mcs.workspace(shape, mcs.MCS_OP_SPARSE)
    idx = _lists(B, H, N, K, 88)
    # pack: an index out of range, then two lists out of order
    for bad in (lambda a: a.__setitem__((0, 0, 1, 3), N), lambda a: a.__setitem__((0, 0, 2, 5), a[0, 0, 2, 4])):
        x = idx.copy()
        bad(x)
        mask = torch.zeros(B, H, G, W, dtype=torch.int32, device="cuda")
        mcs.mcs_meta_pack(shape, torch.from_numpy(x).cuda(), mask, ws)
        st, info = mcs.mcs_poll_status(ws)
        assert st == 5, info  # MCS_ERR_BAD_INDEX
    # unpack: one bit too many, one bit too few, a bit at a position >= N
    good = oracle.meta_pack(idx, N)
    variants = []
    m = good.copy()
    free = next(b for b in range(32) if not (int(m[0, 0, 0, 0]) >> b) & 1)
    m[0, 0, 0, 0] |= np.uint32(1 << free)
    variants.append(m)
    m = good.copy()
    w = int(np.nonzero(m[0, 0, 1])[0][0])
    low = int(m[0, 0, 1, w]) & -int(m[0, 0, 1, w])
    m[0, 0, 1, w] = np.uint32(int(m[0, 0, 1, w]) ^ low)
    variants.append(m)
    m = good.copy()
    m[0, 0, 2, W - 1] |= np.uint32(1 << 31)  # N = 500: bit 31 of the last word is position 511
    variants.append(m)
    n_out = B * H * G * K
    for m in variants:
        buf = torch.full((n_out + 64,), -3, dtype=torch.int32, device="cuda")
        mcs.mcs_meta_unpack(shape, torch.from_numpy(m.view(np.int32)).cuda(), buf[:n_out], ws)
        st, info = mcs.mcs_poll_status(ws)
        assert st == 5, info
        assert torch.all(buf[n_out:] == -3)  # nothing written past the destination
    with pytest.raises(mcs.MCSError):
        mcs.mcs_meta_pack(shape, None, torch.zeros(1, dtype=torch.int32, device="cuda"), ws)
    with pytest.raises(mcs.MCSError):
        mcs.mcs_meta_unpack(mcs.Shape(B, H, N, 64, topk=0), torch.zeros(1, dtype=torch.int32, device="cuda"),
                            torch.zeros(1, dtype=torch.int32, device="cuda"), ws)
