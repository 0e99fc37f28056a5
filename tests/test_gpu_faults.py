"""Error paths of the C ABI on the GPU, all raised on the host or by bounded
device waits (no GPU fault is provoked): argument validation, planted
out-of-range indices, and a producer that never delivers (forced timeout)."""
import pytest

import synth
from helpers import to_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mcs():
    import free_sparse_attention_pddp_b200 as m

    m.load()
    return m


def _small(N=512, H=1, d=64, K=64):
    w = synth.small(N, H=H, d=d, seed=5)
    q, k, v = (to_dev(synth.generate(w, t)) for t in "qkv")
    perm = torch.arange(N, dtype=torch.int32, device="cuda").repeat(1, H, 1).contiguous()
    G = (N + 127) // 128
    idx = torch.arange(K, dtype=torch.int32, device="cuda").repeat(1, H, G, 1).contiguous()
    return q, k, v, perm, idx


def test_invalid_arguments_enqueue_nothing(mcs):
    q, k, v, perm, idx = _small()
    shape = mcs.Shape(1, 1, 512, 64, topk=64)
    o = torch.empty_like(q)
    ws = mcs.workspace(shape, mcs.MCS_OP_SPARSE)
    with pytest.raises(mcs.MCSError) as e:
        mcs.mcs_sparse(shape, None, k, v, perm, idx, None, o, ws)
    assert e.value.code == 1
    with pytest.raises(mcs.MCSError) as e:  # misaligned pointer
        mcs.mcs_sparse(shape, q.view(-1)[1:], k, v, perm, idx, None, o, ws)
    assert e.value.code == 1
    with pytest.raises(mcs.MCSError) as e:  # workspace too small
        mcs.mcs_sparse(shape, q, k, v, perm, idx, None, o, ws[:16])
    assert e.value.code == 1
    bad = mcs.Shape(1, 1, 512, 96, topk=64)
    with pytest.raises(mcs.MCSError) as e:
        mcs.mcs_dense(bad, q, k, v, o, None, ws)
    assert e.value.code == 2
    with pytest.raises(mcs.MCSError):
        mcs.mcs_anchor(shape, q, k, v, perm, o, idx, torch.empty(1, 1, 512, 64, dtype=torch.bfloat16, device="cuda"),
                       None, ws)  # workspace sized for the sparse op, too small for the anchor
    assert mcs.mcs_poll_status(ws)[0] == 0


def test_out_of_range_index_is_reported(mcs):
    q, k, v, perm, idx = _small()
    shape = mcs.Shape(1, 1, 512, 64, topk=64)
    o = torch.empty_like(q)
    ws = mcs.workspace(shape, mcs.MCS_OP_SPARSE)
    idx[0, 0, 1, 5] = 512  # one past the end
    mcs.mcs_sparse(shape, q, k, v, perm, idx, None, o, ws)
    st, info = mcs.mcs_poll_status(ws)
    assert st == 5 and info[1] == 512
    perm[0, 0, 3] = -7
    idx[0, 0, 1, 5] = 5
    mcs.mcs_sparse(shape, q, k, v, perm, idx, None, o, ws)
    st, info = mcs.mcs_poll_status(ws)
    assert st == 5 and info[1] == -7
    # the status was cleared by the poll; a clean call reports OK
    perm[0, 0, 3] = 3
    mcs.mcs_sparse(shape, q, k, v, perm, idx, None, o, ws)
    assert mcs.mcs_poll_status(ws)[0] == 0


def test_forced_timeout_is_reported_and_context_survives(mcs):
    from free_sparse_attention_pddp_b200.binding import debug_set_flags

    q, k, v, perm, idx = _small(N=256, K=200)
    shape = mcs.Shape(1, 1, 256, 64, topk=200)
    o = torch.empty_like(q)
    ws = mcs.workspace(shape, mcs.MCS_OP_SPARSE)
    debug_set_flags(1)
    try:
        mcs.mcs_sparse(shape, q, k, v, perm, idx, None, o, ws)
        st, info = mcs.mcs_poll_status(ws)
    finally:
        debug_set_flags(0)
    assert st == 4, (st, info)
    # the CUDA context is still usable: a normal call succeeds
    mcs.mcs_sparse(shape, q, k, v, perm, idx, None, o, ws)
    assert mcs.mcs_poll_status(ws)[0] == 0
    assert torch.isfinite(o.float()).all()


def test_forced_timeout_in_dense_pair_kernel(mcs):
    """mcs_dense at d = 128 (the kernel over pairs of query tiles): with the
    first K/V tile never delivered, the bounded waits expire, the status block
    reports MCS_ERR_TIMEOUT and a following call succeeds."""
    from free_sparse_attention_pddp_b200.binding import debug_set_flags

    N, d = 640, 128
    g = torch.Generator(device="cpu").manual_seed(5)
    q, k, v = (torch.randn(1, N, 1, d, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    shape = mcs.Shape(1, 1, N, d)
    o = torch.empty_like(q)
    ws = mcs.workspace(shape, mcs.MCS_OP_DENSE)
    debug_set_flags(1)
    try:
        mcs.mcs_dense(shape, q, k, v, o, None, ws)
        st, info = mcs.mcs_poll_status(ws)
    finally:
        debug_set_flags(0)
    assert st == 4, (st, info)
    mcs.mcs_dense(shape, q, k, v, o, None, ws)
    assert mcs.mcs_poll_status(ws)[0] == 0
    assert torch.isfinite(o.float()).all()
