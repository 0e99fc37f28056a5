"""ctypes binding of libmcs.so with the C ABI's names (argument marshalling only).

Every function takes torch tensors (device memory) and enqueues on the current
CUDA stream unless a stream is given. Errors returned by the library raise
``MCSError``.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(HERE, "libmcs.so")
_lib = None

MCS_GROUP_SIZE = 128
MCS_INFO_WORDS = 8
MCS_OP_GROUP, MCS_OP_ANCHOR, MCS_OP_SPARSE, MCS_OP_DENSE = 0, 1, 2, 3


class MCSError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {mcs_status_string(code)} ({code})")
        self.code = code


class Shape(ctypes.Structure):
    """mcs_shape: B, H, N, d, group, topk, scale (scale <= 0 selects 1/sqrt(d))."""

    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int), ("d", ctypes.c_int),
                ("group", ctypes.c_int), ("topk", ctypes.c_int), ("scale", ctypes.c_float)]

    def __init__(self, B, H, N, d, topk=0, scale=0.0, group=MCS_GROUP_SIZE):
        super().__init__(B, H, N, d, group, topk, scale)


def lib_path() -> str:
    return _LIB_PATH


def load():
    """Load libmcs.so from this package directory (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise OSError(f"{_LIB_PATH} is missing: build it with `python -m free_sparse_attention_pddp_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, sz, sp = ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(Shape)
    lib.mcs_workspace_bytes.restype = sz
    lib.mcs_workspace_bytes.argtypes = [sp, ctypes.c_int]
    lib.mcs_meta_mask_bytes.restype = sz
    lib.mcs_meta_mask_bytes.argtypes = [sp]
    for name, args in [
        ("mcs_group", [sp, vp, vp, vp, sz, vp]),
        ("mcs_group_fast", [sp, vp, vp, ctypes.c_int, vp, sz, vp]),
        ("mcs_group_ex", [sp, vp, vp, ctypes.c_int, ctypes.c_int, vp, sz, vp]),
        ("mcs_anchor", [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, vp]),
        ("mcs_sparse", [sp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        ("mcs_sparse_noalloc", [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        ("mcs_dense", [sp, vp, vp, vp, vp, vp, vp, sz, vp]),
        ("mcs_sparse_host", [sp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int, vp, sz, vp, vp, vp]),
        ("mcs_meta_copy", [vp, vp, sz, ctypes.c_int, vp, vp, vp]),
        ("mcs_meta_pack", [sp, vp, vp, vp, sz, vp]),
        ("mcs_meta_unpack", [sp, vp, vp, vp, sz, vp]),
        ("mcs_poll_status", [vp, vp, vp]),
    ]:
        f = getattr(lib, name)
        f.restype = ctypes.c_int
        f.argtypes = args
    lib.mcs_status_string.restype = ctypes.c_char_p
    lib.mcs_status_string.argtypes = [ctypes.c_int]
    lib.mcs_debug_set_flags.restype = None
    lib.mcs_debug_set_flags.argtypes = [ctypes.c_int]
    lib.mcs_debug_launch_count.restype = ctypes.c_longlong
    lib.mcs_debug_launch_count.argtypes = []
    lib.mcs_debug_set_anchor_chunk_events.restype = None
    lib.mcs_debug_set_anchor_chunk_events.argtypes = [vp, ctypes.c_int]
    _lib = lib
    return lib


def mcs_status_string(code: int) -> str:
    return load().mcs_status_string(int(code)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch

        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(code: int, what: str):
    if code != 0:
        raise MCSError(code, what)


def mcs_workspace_bytes(shape: Shape, op: int) -> int:
    return int(load().mcs_workspace_bytes(ctypes.byref(shape), op))


def workspace(shape: Shape, op: int, device="cuda"):
    """Allocate a zeroed workspace of the size the library asks for (uint8 torch tensor)."""
    import torch

    n = mcs_workspace_bytes(shape, op)
    if n == 0:
        raise MCSError(1, "mcs_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def mcs_group(shape, q, perm, ws, stream=None):
    _check(load().mcs_group(ctypes.byref(shape), _ptr(q), _ptr(perm), _ptr(ws), ws.numel(), _stream(stream)),
           "mcs_group")


def mcs_group_fast(shape, q, perm, krylov_steps, ws, stream=None):
    """Fast PDDP grouping: split directions from a fixed number of Lanczos steps."""
    _check(load().mcs_group_fast(ctypes.byref(shape), _ptr(q), _ptr(perm), int(krylov_steps), _ptr(ws), ws.numel(),
                                 _stream(stream)), "mcs_group_fast")


MCS_GROUP_WHITEN = 1


def mcs_group_ex(shape, q, perm, ws, krylov_steps=0, whiten=False, stream=None):
    """Grouping with options: krylov_steps (0 = converged direction) and per-channel whitening."""
    _check(load().mcs_group_ex(ctypes.byref(shape), _ptr(q), _ptr(perm), int(krylov_steps),
                               MCS_GROUP_WHITEN if whiten else 0, _ptr(ws), ws.numel(), _stream(stream)),
           "mcs_group_ex")


def mcs_anchor(shape, q, k, v, perm, o, kv_idx, resid, lse, ws, stream=None, stage_events=None):
    ev = None
    if stage_events is not None:
        if len(stage_events) != 5:
            raise ValueError("stage_events needs 5 events")
        for e in stage_events:
            if e.cuda_event == 0:  # torch creates the CUDA event lazily, on first record
                e.record()
        arr = (ctypes.c_void_p * 5)(*[e.cuda_event for e in stage_events])
        ev = ctypes.cast(arr, ctypes.c_void_p)
    _check(load().mcs_anchor(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(perm), _ptr(o), _ptr(kv_idx),
                             _ptr(resid), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream), ev), "mcs_anchor")


def mcs_sparse(shape, q, k, v, perm, kv_idx, resid, o, ws, stream=None):
    _check(load().mcs_sparse(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(perm), _ptr(kv_idx),
                             _ptr(resid), _ptr(o), _ptr(ws), ws.numel(), _stream(stream)), "mcs_sparse")


def mcs_sparse_noalloc(shape, q, k, v, perm, kv_idx, resid, o, stream=None, report=True):
    """Reuse step without a workspace (static device scratch; see include/mcs.h).

    With report=True the call waits for the stream and returns the info words;
    otherwise it only enqueues and returns None.
    """
    info = (ctypes.c_int32 * MCS_INFO_WORDS)() if report else None
    _check(load().mcs_sparse_noalloc(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(perm), _ptr(kv_idx),
                                     _ptr(resid), _ptr(o), ctypes.cast(info, ctypes.c_void_p) if report else None,
                                     _stream(stream)), "mcs_sparse_noalloc")
    return list(info) if report else None


def mcs_sparse_host(shape, q_host, k_host, v_host, perm, kv_idx, resid, o_host, q_dev, k_dev, v_dev, o_dev,
                    head_chunks, ws, stream, copy_in, copy_out):
    """Reuse step on host q/k/v/o, head chunks pipelined over three streams (see include/mcs.h)."""
    _check(load().mcs_sparse_host(ctypes.byref(shape), _ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(perm),
                                  _ptr(kv_idx), _ptr(resid), _ptr(o_host), _ptr(q_dev), _ptr(k_dev), _ptr(v_dev),
                                  _ptr(o_dev), int(head_chunks), _ptr(ws), ws.numel(), _stream(stream),
                                  _stream(copy_in), _stream(copy_out)), "mcs_sparse_host")


def mcs_dense(shape, q, k, v, o, lse, ws, stream=None):
    _check(load().mcs_dense(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(ws),
                            ws.numel(), _stream(stream)), "mcs_dense")


def _event(ev, must_exist: bool):
    """Raw handle of a torch.cuda.Event (None for None). torch creates the CUDA
    event lazily on its first record; an event that must exist is recorded once
    first (waiting on a never-recorded event is a no-op, so it may stay null)."""
    if ev is None:
        return None
    if ev.cuda_event == 0:
        if not must_exist:
            return None
        ev.record()
    return ctypes.c_void_p(ev.cuda_event)


def mcs_meta_copy(dst, src, nbytes: int, to_host: bool, side_stream, wait_event=None, done_event=None):
    """Copy metadata on `side_stream`: wait for `wait_event`, copy, record `done_event`."""
    _check(load().mcs_meta_copy(_ptr(dst), _ptr(src), nbytes, int(to_host), _stream(side_stream),
                                _event(wait_event, False), _event(done_event, True)), "mcs_meta_copy")


def mcs_meta_mask_bytes(shape: Shape) -> int:
    """Bytes of the packed selection (uint32 [B, H, G, ceil(N/32)]); 0 for an invalid shape."""
    return int(load().mcs_meta_mask_bytes(ctypes.byref(shape)))


def mcs_meta_pack(shape, kv_idx, mask, ws, stream=None):
    """kv_idx [B,H,G,K] ascending -> packed selection mask (device to device)."""
    _check(load().mcs_meta_pack(ctypes.byref(shape), _ptr(kv_idx), _ptr(mask), _ptr(ws), ws.numel(),
                                _stream(stream)), "mcs_meta_pack")


def mcs_meta_unpack(shape, mask, kv_idx, ws, stream=None):
    """Packed selection mask -> kv_idx [B,H,G,K] ascending (device to device)."""
    _check(load().mcs_meta_unpack(ctypes.byref(shape), _ptr(mask), _ptr(kv_idx), _ptr(ws), ws.numel(),
                                  _stream(stream)), "mcs_meta_unpack")


def mcs_poll_status(ws, stream=None):
    """Synchronise, read and clear the status block: returns (status, info words)."""
    info = (ctypes.c_int32 * MCS_INFO_WORDS)()
    code = load().mcs_poll_status(_ptr(ws), ctypes.cast(info, ctypes.c_void_p), _stream(stream))
    return int(code), list(info)


def debug_set_flags(flags: int):
    """Test hook (include/mcs_test.h): process-wide debug flags."""
    load().mcs_debug_set_flags(int(flags))


_chunk_event_handles = None


def debug_set_anchor_chunk_events(events):
    """Measurement hook (include/mcs_test.h): record `events` (torch.cuda.Event
    with timing, 3 per head chunk) around each chunk's mass and top-K launches
    of later mcs_anchor calls; None turns it off."""
    global _chunk_event_handles
    if events is None:
        _chunk_event_handles = None
        load().mcs_debug_set_anchor_chunk_events(None, 0)
        return
    for e in events:
        if e.cuda_event == 0:  # created lazily by torch on first record
            e.record()
    _chunk_event_handles = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    load().mcs_debug_set_anchor_chunk_events(ctypes.cast(_chunk_event_handles, ctypes.c_void_p), len(events))


def debug_launch_count() -> int:
    """Diagnostic hook (include/mcs_test.h): kernel launches enqueued by the library so far."""
    return int(load().mcs_debug_launch_count())
