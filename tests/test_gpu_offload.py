"""Metadata offload and one-layer-ahead prefetch (aiwillknow analysis, step 5;
paper Table 8) through mcs_meta_copy.

After the anchor step every layer's KV indices and residual R go to pinned
host memory; during the reuse steps layer l+1's metadata comes back on a side
stream while layer l computes, into one of two device buffers. The pipeline's
outputs must equal, bit for bit, the reuse step run with every layer's
metadata resident on the device: any ordering fault (a buffer overwritten
while a kernel still reads it, or read before its copy landed) changes them.
"""
import numpy as np
import pytest

import synth
from helpers import to_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

LAYERS, B, N, H, D, DENSITY, SEED = 3, 1, 2048, 2, 64, 0.15, 4242


@pytest.fixture(scope="module")
def mcs():
    import free_sparse_attention_pddp_b200 as m

    m.load()
    return m


def _layer_inputs(w, layer, step):
    return [to_dev(synth.generate(w, t, step, layer)) for t in "qkv"]


@pytest.fixture(scope="module")
def anchored(mcs):
    """Per layer: fresh inputs, grouping and anchor on step 0; reuse inputs of step 1."""
    w = synth.small(N, H=H, d=D, density=DENSITY, seed=SEED, B=B)
    K = synth.topk_for(N, DENSITY)
    G = (N + 127) // 128
    shape = mcs.Shape(B, H, N, D, topk=K)
    ws = {op: mcs.workspace(shape, op) for op in (mcs.MCS_OP_GROUP, mcs.MCS_OP_ANCHOR, mcs.MCS_OP_SPARSE)}
    layers = []
    for layer in range(LAYERS):
        q0, k0, v0 = _layer_inputs(w, layer, 0)
        perm = torch.empty(B, H, N, dtype=torch.int32, device="cuda")
        idx = torch.empty(B, H, G, K, dtype=torch.int32, device="cuda")
        resid = torch.empty(B, H, N, D, dtype=torch.bfloat16, device="cuda")
        o0 = torch.empty(B, N, H, D, dtype=torch.bfloat16, device="cuda")
        mcs.mcs_group(shape, q0, perm, ws[mcs.MCS_OP_GROUP])
        mcs.mcs_anchor(shape, q0, k0, v0, perm, o0, idx, resid, None, ws[mcs.MCS_OP_ANCHOR])
        layers.append(dict(perm=perm, idx=idx, resid=resid, qkv=_layer_inputs(w, layer, 1)))
    for wsx in ws.values():
        st, info = mcs.mcs_poll_status(wsx)
        assert st == 0, info
    return shape, ws, layers


def _as_bytes(t):
    return t.view(torch.uint8).view(-1)


def test_meta_copy_round_trip_is_exact(mcs, anchored):
    shape, ws, layers = anchored
    side = torch.cuda.Stream()
    after_anchor = torch.cuda.Event()
    after_anchor.record()  # on the compute stream, after every anchor above
    for L in layers:
        for name in ("idx", "resid"):
            dev = L[name]
            host = torch.empty(dev.numel() * dev.element_size(), dtype=torch.uint8, pin_memory=True)
            copied = torch.cuda.Event()
            mcs.mcs_meta_copy(host, dev, host.numel(), True, side, wait_event=after_anchor, done_event=copied)
            copied.synchronize()
            back = torch.zeros_like(_as_bytes(dev))
            landed = torch.cuda.Event()
            mcs.mcs_meta_copy(back, host, host.numel(), False, side, done_event=landed)
            landed.synchronize()
            assert torch.equal(back, _as_bytes(dev)), name


def test_one_layer_ahead_prefetch_matches_resident_metadata(mcs, anchored):
    shape, ws, layers = anchored
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    sparse_ws = ws[mcs.MCS_OP_SPARSE]

    # reference: every layer's metadata resident on the device
    want = []
    for L in layers:
        o = torch.empty(B, N, H, D, dtype=torch.bfloat16, device="cuda")
        mcs.mcs_sparse(shape, *L["qkv"], L["perm"], L["idx"], L["resid"], o, sparse_ws)
        want.append(o)

    # offload: D2H of every layer's metadata after the anchor, on the side stream
    ready = torch.cuda.Event()
    ready.record(main)
    host = []
    for L in layers:
        h = {}
        for name in ("idx", "resid"):
            h[name] = torch.empty(L[name].numel() * L[name].element_size(), dtype=torch.uint8, pin_memory=True)
            mcs.mcs_meta_copy(h[name], L[name], h[name].numel(), True, side, wait_event=ready)
        host.append(h)
    offloaded = torch.cuda.Event()
    offloaded.record(side)
    offloaded.synchronize()

    # two device buffers; the first reuse kernel must not see stale contents
    bufs = [{name: torch.full_like(layers[0][name], 0 if name == "resid" else -1) for name in ("idx", "resid")}
            for _ in range(2)]
    landed = [torch.cuda.Event() for _ in range(2)]
    freed = [torch.cuda.Event() for _ in range(2)]

    def prefetch(layer):
        slot = bufs[layer % 2]
        for name in ("idx", "resid"):
            nbytes = host[layer][name].numel()
            # wait until the layer that last read this buffer has finished
            mcs.mcs_meta_copy(_as_bytes(slot[name]), host[layer][name], nbytes, False, side,
                              wait_event=freed[layer % 2], done_event=landed[layer % 2] if name == "resid" else None)

    got = []
    prefetch(0)
    for layer, L in enumerate(layers):
        main.wait_event(landed[layer % 2])
        if layer + 1 < LAYERS:
            prefetch(layer + 1)  # overlaps this layer's compute
        o = torch.empty(B, N, H, D, dtype=torch.bfloat16, device="cuda")
        slot = bufs[layer % 2]
        mcs.mcs_sparse(shape, *L["qkv"], L["perm"], slot["idx"], slot["resid"], o, sparse_ws, stream=main)
        freed[layer % 2].record(main)
        got.append(o)
    st, info = mcs.mcs_poll_status(sparse_ws)
    assert st == 0, info
    for layer in range(LAYERS):
        assert torch.equal(got[layer].view(torch.int16), want[layer].view(torch.int16)), f"layer {layer}"


def test_packed_prefetch_matches_resident_metadata(mcs, anchored):
    """The same pipeline with the selection packed into N-bit masks: pack after the
    anchor, offload masks and R, and on the side stream copy them back and unpack
    into the slot's index buffer before the layer's reuse step."""
    shape, ws, layers = anchored
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    sparse_ws = ws[mcs.MCS_OP_SPARSE]
    side_ws = mcs.workspace(shape, mcs.MCS_OP_SPARSE)
    mbytes = mcs.mcs_meta_mask_bytes(shape)
    want = []
    for L in layers:
        o = torch.empty(B, N, H, D, dtype=torch.bfloat16, device="cuda")
        mcs.mcs_sparse(shape, *L["qkv"], L["perm"], L["idx"], L["resid"], o, sparse_ws)
        want.append(o)
    masks = [torch.empty(mbytes, dtype=torch.uint8, device="cuda") for _ in layers]
    for L, m in zip(layers, masks):
        mcs.mcs_meta_pack(shape, L["idx"], m, sparse_ws)
    ready = torch.cuda.Event()
    ready.record(main)
    host = []
    for L, m in zip(layers, masks):
        h = {"mask": torch.empty(mbytes, dtype=torch.uint8, pin_memory=True),
             "resid": torch.empty(L["resid"].numel() * 2, dtype=torch.uint8, pin_memory=True)}
        mcs.mcs_meta_copy(h["mask"], m, mbytes, True, side, wait_event=ready)
        mcs.mcs_meta_copy(h["resid"], L["resid"], h["resid"].numel(), True, side, wait_event=ready)
        host.append(h)
    offloaded = torch.cuda.Event()
    offloaded.record(side)
    offloaded.synchronize()
    bufs = [{"mask": torch.zeros(mbytes, dtype=torch.uint8, device="cuda"),
             "idx": torch.full_like(layers[0]["idx"], -1), "resid": torch.zeros_like(layers[0]["resid"])}
            for _ in range(2)]
    landed = [torch.cuda.Event() for _ in range(2)]
    freed = [torch.cuda.Event() for _ in range(2)]
    side.wait_stream(main)  # the buffer fills above land first

    def prefetch(layer):
        slot = bufs[layer % 2]
        mcs.mcs_meta_copy(slot["mask"], host[layer]["mask"], mbytes, False, side, wait_event=freed[layer % 2])
        mcs.mcs_meta_copy(_as_bytes(slot["resid"]), host[layer]["resid"], host[layer]["resid"].numel(), False, side)
        mcs.mcs_meta_unpack(shape, slot["mask"], slot["idx"], side_ws, side)
        landed[layer % 2].record(side)

    got = []
    prefetch(0)
    for layer, L in enumerate(layers):
        main.wait_event(landed[layer % 2])
        if layer + 1 < LAYERS:
            prefetch(layer + 1)
        o = torch.empty(B, N, H, D, dtype=torch.bfloat16, device="cuda")
        slot = bufs[layer % 2]
        mcs.mcs_sparse(shape, *L["qkv"], L["perm"], slot["idx"], slot["resid"], o, sparse_ws, stream=main)
        freed[layer % 2].record(main)
        got.append(o)
    for wsx in (sparse_ws, side_ws):
        st, info = mcs.mcs_poll_status(wsx)
        assert st == 0, info
    for layer in range(LAYERS):
        assert torch.equal(got[layer].view(torch.int16), want[layer].view(torch.int16)), f"layer {layer}"


def test_meta_copy_arguments(mcs):
    side = torch.cuda.Stream()
    x = torch.zeros(16, dtype=torch.uint8, device="cuda")
    mcs.mcs_meta_copy(None, None, 0, True, side)  # zero bytes: nothing enqueued, no error
    with pytest.raises(mcs.MCSError) as e:
        mcs.mcs_meta_copy(None, x, 16, True, side)
    assert e.value.code == 1
    with pytest.raises(mcs.MCSError) as e:
        mcs.mcs_meta_copy(x, None, 16, False, side)
    assert e.value.code == 1
