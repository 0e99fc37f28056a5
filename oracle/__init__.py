"""MC-Sparse CPU oracle (fp64), Python side.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``. The product path (the package
``free_sparse_attention_pddp_b200``) never imports it, and this module never
imports the product path.

The arithmetic lives in ``mcs_oracle.c`` (plain C, double precision, one
(batch, head) slice per call); this file compiles it with gcc, marshals numpy
arrays, and composes per-group calls. ctypes releases the GIL during a foreign
call, so ``threads > 1`` runs groups on several host cores at once.

Tensors are bf16 bit patterns (numpy uint16) in the [B, N, H, d] layout.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mcs_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_i32p = ctypes.POINTER(ctypes.c_int32)
_f64p = ctypes.POINTER(ctypes.c_double)
_u16p = ctypes.POINTER(ctypes.c_uint16)


def build(force: bool = False, src: str | None = None, out: str | None = None) -> str:
    """Compile mcs_oracle.c into a shared library (gcc -O2, strict IEEE fp64).

    ``src``/``out`` let a test build a variant (a copy of the source with a
    planted mistake) into a separate file without touching the default library.
    """
    target = out or _LIB
    if force or out or not os.path.exists(target) or os.path.getmtime(target) < os.path.getmtime(_SRC):
        tmp = target + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", tmp, src or _SRC, "-lm"])
        os.replace(tmp, target)
    return target


def _bind(lib):
    lib.orc_jacobi_eigh.restype = ctypes.c_int
    lib.orc_jacobi_eigh.argtypes = [ctypes.c_int, _f64p, _f64p, _f64p, ctypes.c_double, ctypes.c_int]
    lib.orc_pddp_left_size.restype = ctypes.c_int
    lib.orc_pddp_left_size.argtypes = [ctypes.c_int, ctypes.c_int]
    lib.orc_pddp_split.restype = ctypes.c_int
    lib.orc_pddp_split.argtypes = [_u16p, ctypes.c_long, ctypes.c_int, _i32p, ctypes.c_int, ctypes.c_int, _i32p,
                                   _i32p, _f64p, _f64p, _f64p, _f64p]
    lib.orc_pddp.restype = ctypes.c_int
    lib.orc_pddp.argtypes = [_u16p, ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_int, _i32p, _f64p,
                             ctypes.c_int]
    lib.orc_channel_scale.restype = None
    lib.orc_channel_scale.argtypes = [_u16p, ctypes.c_long, ctypes.c_int, ctypes.c_int, _f64p]
    lib.orc_pddp_split_w.restype = ctypes.c_int
    lib.orc_pddp_split_w.argtypes = [_u16p, ctypes.c_long, ctypes.c_int, _f64p, _i32p, ctypes.c_int, ctypes.c_int,
                                     _i32p, _i32p, _f64p, _f64p, _f64p, _f64p]
    lib.orc_pddp_w.restype = ctypes.c_int
    lib.orc_pddp_w.argtypes = [_u16p, ctypes.c_long, ctypes.c_int, _f64p, ctypes.c_int, ctypes.c_int, _i32p]
    lib.orc_splitmix64.restype = ctypes.c_uint64
    lib.orc_splitmix64.argtypes = [ctypes.c_uint64]
    lib.orc_pddp_split_krylov.restype = ctypes.c_int
    lib.orc_pddp_split_krylov.argtypes = [_u16p, ctypes.c_long, ctypes.c_int, _i32p, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, _i32p, _i32p, _f64p, _f64p, _f64p]
    lib.orc_pddp_krylov.restype = ctypes.c_int
    lib.orc_pddp_krylov.argtypes = [_u16p, ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    _i32p]
    lib.orc_attention_rows.restype = ctypes.c_int
    lib.orc_attention_rows.argtypes = [_u16p, _u16p, _u16p, ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_double, _i32p, ctypes.c_int, _i32p, ctypes.c_int, _f64p, _f64p]
    lib.orc_group_mass.restype = ctypes.c_int
    lib.orc_group_mass.argtypes = [_u16p, _u16p, ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                   _i32p, ctypes.c_int, _f64p]
    lib.orc_topk.restype = ctypes.c_int
    lib.orc_topk.argtypes = [_f64p, ctypes.c_int, ctypes.c_int, _i32p]
    lib.orc_anchor_group.restype = ctypes.c_int
    lib.orc_anchor_group.argtypes = [_u16p, _u16p, _u16p, ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_double, _i32p, ctypes.c_int, ctypes.c_int, _f64p, _f64p, _f64p,
                                     _f64p, _f64p, _i32p]
    lib.orc_reuse_group.restype = ctypes.c_int
    lib.orc_reuse_group.argtypes = [_u16p, _u16p, _u16p, ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_double, _i32p, ctypes.c_int, _i32p, ctypes.c_int, _f64p, _f64p]
    lib.orc_round_bf16.restype = None
    lib.orc_round_bf16.argtypes = [_f64p, ctypes.c_long, _u16p]
    return lib


def load(path: str | None = None):
    """Load (building if needed) the oracle library; ``path`` loads a variant."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _p(a, t):
    return a.ctypes.data_as(t) if a is not None else None


def _head(x: np.ndarray, b: int, h: int):
    """Pointer to token 0 of (b, h) in a contiguous [B, N, H, d] uint16 array, and the token stride."""
    assert x.dtype == np.uint16 and x.flags.c_contiguous and x.ndim == 4
    B, N, H, d = x.shape
    ptr = ctypes.cast(x.ctypes.data + ((b * N * H + h) * d) * 2, _u16p)
    return ptr, H * d


def default_scale(d: int) -> float:
    """Softmax scale 1/sqrt(d) (standard scaled dot-product attention)."""
    return 1.0 / math.sqrt(d)


# ---------------------------------------------------------------------------
# PDDP
# ---------------------------------------------------------------------------

def jacobi_eigh(A: np.ndarray, tol: float = 1e-14, max_sweeps: int = 200, lib=None):
    """Eigenpairs of a symmetric matrix by cyclic Jacobi; descending eigenvalues, eigenvectors as columns."""
    lib = lib or load()
    n = A.shape[0]
    W = np.ascontiguousarray(A, dtype=np.float64).copy()
    ev = np.empty(n)
    V = np.empty((n, n))
    sweeps = lib.orc_jacobi_eigh(n, _p(W, _f64p), _p(ev, _f64p), _p(V, _f64p), tol, max_sweeps)
    return ev, V, sweeps


def pddp_left_size(n: int, g: int) -> int:
    """Queries sent left when a node of n splits: ceil(ceil(n/g)/2) * g."""
    T = (n + g - 1) // g
    return ((T + 1) // 2) * g


def pddp_tree(N: int, g: int):
    """Internal nodes of the grouping tree in preorder: (offset, n, L) into the permutation.

    The tree's shape depends only on N and g, so positions in the final
    permutation identify every node.
    """
    out = []

    def rec(off, n):
        if (n + g - 1) // g <= 1:
            return
        L = pddp_left_size(n, g)
        out.append((off, n, L))
        rec(off, L)
        rec(off + L, n - L)

    rec(0, N)
    return out


def pddp(q: np.ndarray, b: int, h: int, g: int = 128, lib=None):
    """Full Fast-PDDP grouping of head (b, h): returns (perm int32[N], relative eigengaps of internal nodes)."""
    lib = lib or load()
    ptr, stride = _head(q, b, h)
    N, d = q.shape[1], q.shape[3]
    perm = np.empty(N, dtype=np.int32)
    nint = max(1, len(pddp_tree(N, g)))
    gaps = np.zeros(nint)
    rc = lib.orc_pddp(ptr, stride, d, N, g, _p(perm, _i32p), _p(gaps, _f64p), nint)
    if rc != 0:
        raise RuntimeError("oracle PDDP: Jacobi did not converge")
    return perm, gaps[: len(pddp_tree(N, g))]


def channel_scale(q: np.ndarray, b: int, h: int, lib=None) -> np.ndarray:
    """Whitened grouping: 1 / (population std of each channel over head (b, h)'s queries), 1 where it is 0."""
    lib = lib or load()
    ptr, stride = _head(q, b, h)
    N, d = q.shape[1], q.shape[3]
    w = np.empty(d)
    lib.orc_channel_scale(ptr, stride, d, N, _p(w, _f64p))
    return w


def pddp_whitened(q: np.ndarray, b: int, h: int, g: int = 128, lib=None) -> np.ndarray:
    """Grouping of head (b, h) on its per-channel standardised queries: perm int32[N]."""
    lib = lib or load()
    w = channel_scale(q, b, h, lib=lib)
    ptr, stride = _head(q, b, h)
    N, d = q.shape[1], q.shape[3]
    perm = np.empty(N, dtype=np.int32)
    if lib.orc_pddp_w(ptr, stride, d, _p(w, _f64p), N, g, _p(perm, _i32p)) != 0:
        raise RuntimeError("oracle PDDP: Jacobi did not converge")
    return perm


def pddp_split(q: np.ndarray, b: int, h: int, members: np.ndarray, g: int = 128, lib=None, wscale=None):
    """Split one node: returns dict(left, right, dir, proj, split_p, eig). With ``wscale`` (from
    channel_scale) the node is split as in the whitened grouping (dir, proj in whitened coordinates)."""
    lib = lib or load()
    ptr, stride = _head(q, b, h)
    d = q.shape[3]
    members = np.ascontiguousarray(members, dtype=np.int32)
    n = len(members)
    L = lib.orc_pddp_left_size(n, g)  # the library's own rule sizes the buffers it fills
    left = np.empty(L, dtype=np.int32)
    right = np.empty(n - L, dtype=np.int32)
    direc = np.empty(d)
    proj = np.empty(n)
    split_p = np.empty(1)
    eig = np.empty(2)
    if wscale is None:
        rc = lib.orc_pddp_split(ptr, stride, d, _p(members, _i32p), n, g, _p(left, _i32p), _p(right, _i32p),
                                _p(direc, _f64p), _p(proj, _f64p), _p(split_p, _f64p), _p(eig, _f64p))
    else:
        wscale = np.ascontiguousarray(wscale, dtype=np.float64)
        rc = lib.orc_pddp_split_w(ptr, stride, d, _p(wscale, _f64p), _p(members, _i32p), n, g, _p(left, _i32p),
                                  _p(right, _i32p), _p(direc, _f64p), _p(proj, _f64p), _p(split_p, _f64p),
                                  _p(eig, _f64p))
    if rc != 0:
        raise RuntimeError("oracle PDDP split: Jacobi did not converge")
    return dict(left=left, right=right, dir=direc, proj=proj, split_p=float(split_p[0]), eig=eig)


def splitmix64(index: int, lib=None) -> int:
    """Output number ``index`` (1, 2, ...) of SplitMix64 started from state 0."""
    lib = lib or load()
    return int(lib.orc_splitmix64(index))


def pddp_split_krylov(q: np.ndarray, b: int, h: int, members: np.ndarray, k: int, g: int = 128, lib=None):
    """"Fast" split of one node: direction = top Ritz vector on the k-step Krylov space
    of the node's scatter matrix from the SplitMix64 start vector. Returns dict(left, right, dir, proj, split_p)."""
    lib = lib or load()
    ptr, stride = _head(q, b, h)
    d = q.shape[3]
    members = np.ascontiguousarray(members, dtype=np.int32)
    n = len(members)
    L = lib.orc_pddp_left_size(n, g)  # the library's own rule sizes the buffers it fills
    left = np.empty(L, dtype=np.int32)
    right = np.empty(n - L, dtype=np.int32)
    direc = np.empty(d)
    proj = np.empty(n)
    split_p = np.empty(1)
    rc = lib.orc_pddp_split_krylov(ptr, stride, d, _p(members, _i32p), n, g, k, _p(left, _i32p), _p(right, _i32p),
                                   _p(direc, _f64p), _p(proj, _f64p), _p(split_p, _f64p))
    if rc != 0:
        raise RuntimeError("oracle Krylov split: Jacobi did not converge")
    return dict(left=left, right=right, dir=direc, proj=proj, split_p=float(split_p[0]))


def pddp_krylov(q: np.ndarray, b: int, h: int, k: int, g: int = 128, lib=None) -> np.ndarray:
    """Full "fast" grouping of head (b, h) with k Krylov steps per node: perm int32[N]."""
    lib = lib or load()
    ptr, stride = _head(q, b, h)
    N, d = q.shape[1], q.shape[3]
    perm = np.empty(N, dtype=np.int32)
    if lib.orc_pddp_krylov(ptr, stride, d, N, g, k, _p(perm, _i32p)) != 0:
        raise RuntimeError("oracle Krylov PDDP: Jacobi did not converge")
    return perm


# ---------------------------------------------------------------------------
# attention, mass, top-K, anchor, reuse
# ---------------------------------------------------------------------------

def attention_rows(q, k, v, b, h, rows, keys=None, scale=None, lib=None):
    """fp64 attention of query tokens ``rows`` over ``keys`` (all tokens if None): (o [n,d], lse [n])."""
    lib = lib or load()
    qp, stride = _head(q, b, h)
    kp, _ = _head(k, b, h)
    vp, _ = _head(v, b, h)
    N, d = q.shape[1], q.shape[3]
    scale = default_scale(d) if scale is None else scale
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    keys_a = None if keys is None else np.ascontiguousarray(keys, dtype=np.int32)
    o = np.empty((len(rows), d))
    lse = np.empty(len(rows))
    lib.orc_attention_rows(qp, kp, vp, stride, d, N, scale, _p(rows, _i32p), len(rows),
                           _p(keys_a, _i32p) if keys_a is not None else None,
                           0 if keys_a is None else len(keys_a), _p(o, _f64p), _p(lse, _f64p))
    return o, lse


def group_mass(q, k, b, h, rows, scale=None, lib=None):
    """fp64 group attention mass m(j) = sum_{i in rows} p_ij over all N keys."""
    lib = lib or load()
    qp, stride = _head(q, b, h)
    kp, _ = _head(k, b, h)
    N, d = q.shape[1], q.shape[3]
    scale = default_scale(d) if scale is None else scale
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    mass = np.empty(N)
    lib.orc_group_mass(qp, kp, stride, d, N, scale, _p(rows, _i32p), len(rows), _p(mass, _f64p))
    return mass


def topk(mass: np.ndarray, K: int, lib=None) -> np.ndarray:
    """K largest masses, ties to the lower index, ascending indices (int32)."""
    lib = lib or load()
    mass = np.ascontiguousarray(mass, dtype=np.float64)
    idx = np.empty(K, dtype=np.int32)
    if lib.orc_topk(_p(mass, _f64p), len(mass), K, _p(idx, _i32p)) != 0:
        raise ValueError("K out of range")
    return idx


def anchor_group(q, k, v, b, h, rows, K, scale=None, lib=None):
    """Anchor step for one group: dict(o_dense, o_sparse, resid, lse, mass, idx)."""
    lib = lib or load()
    qp, stride = _head(q, b, h)
    kp, _ = _head(k, b, h)
    vp, _ = _head(v, b, h)
    N, d = q.shape[1], q.shape[3]
    scale = default_scale(d) if scale is None else scale
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    n = len(rows)
    r = dict(o_dense=np.empty((n, d)), o_sparse=np.empty((n, d)), resid=np.empty((n, d)), lse=np.empty(n),
             mass=np.empty(N), idx=np.empty(K, dtype=np.int32))
    rc = lib.orc_anchor_group(qp, kp, vp, stride, d, N, scale, _p(rows, _i32p), n, K, _p(r["o_dense"], _f64p),
                              _p(r["o_sparse"], _f64p), _p(r["resid"], _f64p), _p(r["lse"], _f64p),
                              _p(r["mass"], _f64p), _p(r["idx"], _i32p))
    if rc != 0:
        raise ValueError("K out of range")
    return r


def reuse_group(q, k, v, b, h, rows, idx, resid=None, scale=None, lib=None):
    """Reuse step for one group: sparse attention over ``idx`` plus the residual (fp64, [n, d])."""
    lib = lib or load()
    qp, stride = _head(q, b, h)
    kp, _ = _head(k, b, h)
    vp, _ = _head(v, b, h)
    N, d = q.shape[1], q.shape[3]
    scale = default_scale(d) if scale is None else scale
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    res = None if resid is None else np.ascontiguousarray(resid, dtype=np.float64)
    o = np.empty((len(rows), d))
    lib.orc_reuse_group(qp, kp, vp, stride, d, N, scale, _p(rows, _i32p), len(rows), _p(idx, _i32p), len(idx),
                        _p(res, _f64p) if res is not None else None, _p(o, _f64p))
    return o


def round_bf16(x: np.ndarray, lib=None) -> np.ndarray:
    """Round float64 values to bf16 bit patterns (nearest, ties to even)."""
    lib = lib or load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    lib.orc_round_bf16(_p(x, _f64p), x.size, _p(out, _u16p))
    return out


def groups_of(perm: np.ndarray, g: int = 128):
    """Split a permutation into its groups of g consecutive entries (last may be short)."""
    return [perm[i:i + g] for i in range(0, len(perm), g)]


def run_groups(fn, jobs, threads: int = 1):
    """Map ``fn`` over ``jobs`` on ``threads`` host threads (ctypes drops the GIL)."""
    if threads <= 1:
        return [fn(j) for j in jobs]
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(fn, jobs))


def metadata_bytes(N: int, H: int, d: int, K: int, g: int = 128) -> dict:
    """Per-layer metadata volume of the cached format: bf16 residual [H, N, d] and int32 KV indices [H, G, K].

    The paper's Table 8 counts G as N/g (fractional); ``G_exact`` uses ceil(N/g),
    the number of stored index lists.
    """
    resid = N * H * d * 2
    idx_frac = (N / g) * H * K * 4
    idx_exact = ((N + g - 1) // g) * H * K * 4
    return dict(resid=resid, idx=idx_frac, idx_exact=idx_exact, total=resid + idx_frac,
                total_exact=resid + idx_exact)


def meta_pack(idx: np.ndarray, N: int) -> np.ndarray:
    """Packed selection (the metadata-offload format): for each index list on the
    last axis, ceil(N/32) uint32 words in which bit (j mod 32) of word floor(j/32)
    is set exactly when key j is in the list.

    A restatement of set membership (paper Table 8 counts the selection as int32
    lists; the packed form is the library's), written with numpy's unbuffered OR.
    """
    idx = np.asarray(idx, dtype=np.int64)
    W = (N + 31) // 32
    flat = idx.reshape(-1, idx.shape[-1])
    out = np.zeros((flat.shape[0], W), dtype=np.uint32)
    rows = np.repeat(np.arange(flat.shape[0]), flat.shape[1])
    j = flat.reshape(-1)
    np.bitwise_or.at(out, (rows, j // 32), (np.uint32(1) << (j % 32).astype(np.uint32)).astype(np.uint32))
    return out.reshape(idx.shape[:-1] + (W,))


def meta_unpack(words: np.ndarray, N: int) -> np.ndarray:
    """Inverse of meta_pack: for each row of words, the ascending keys j < N whose
    bit is set. Every row must hold the same number of keys (a selection of K)."""
    words = np.asarray(words, dtype=np.uint32)
    W = words.shape[-1]
    flat = words.reshape(-1, W)
    bits = ((flat[:, :, None] >> np.arange(32, dtype=np.uint32)) & np.uint32(1)).reshape(flat.shape[0], W * 32)
    lists = [np.nonzero(bits[r, :N])[0].astype(np.int32) for r in range(flat.shape[0])]
    K = len(lists[0]) if lists else 0
    if any(len(x) != K for x in lists):
        raise ValueError("rows hold different numbers of keys")
    return np.stack(lists).reshape(words.shape[:-1] + (K,)) if lists else np.zeros(words.shape[:-1] + (0,), np.int32)
