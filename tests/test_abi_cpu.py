"""The C ABI library loads on a machine without a GPU and exports every symbol
the public headers declare; host-only entry points behave as documented."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")


def declared_functions():
    names = []
    for fn in sorted(os.listdir(INCLUDE)):
        if fn.endswith(".h"):
            text = open(os.path.join(INCLUDE, fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(mcs_[a-z_]+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from free_sparse_attention_pddp_b200 import build

    build.build()
    import free_sparse_attention_pddp_b200 as m

    return m.load()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"mcs_group", "mcs_anchor", "mcs_sparse", "mcs_dense", "mcs_meta_copy", "mcs_poll_status",
            "mcs_status_string", "mcs_workspace_bytes"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    import free_sparse_attention_pddp_b200 as m

    assert m.mcs_status_string(0) == "MCS_OK"
    assert m.mcs_status_string(4) == "MCS_ERR_TIMEOUT"
    assert m.mcs_status_string(99) == "MCS_ERR_UNKNOWN"


def test_workspace_sizes(lib):
    import free_sparse_attention_pddp_b200 as m

    s = m.Shape(1, 40, 75600, 128, topk=15120)
    assert m.mcs_workspace_bytes(s, m.MCS_OP_SPARSE) == 256
    assert m.mcs_workspace_bytes(s, m.MCS_OP_DENSE) == 256
    a = m.mcs_workspace_bytes(s, m.MCS_OP_ANCHOR)
    # O_dense fp32 + lse (fp32 hi and lo parts) + queries in group order
    # (bf16), all padded to 591 groups of 128, then a mass chunk of at most 2 GiB
    rows = 40 * 591 * 128
    fixed = rows * 128 * 4 + 2 * rows * 4 + rows * 128 * 2
    assert fixed < a <= fixed + (2 << 30) + 4096
    assert m.mcs_workspace_bytes(s, m.MCS_OP_GROUP) > 40 * 75600 * 12


@pytest.mark.parametrize("bad", [dict(d=96), dict(group=64), dict(topk=0), dict(topk=75601), dict(N=0),
                                 dict(B=0), dict(H=0)])
def test_workspace_rejects_bad_shapes(lib, bad):
    import free_sparse_attention_pddp_b200 as m

    kw = dict(B=1, H=40, N=75600, d=128, topk=15120, group=128)
    kw.update(bad)
    s = m.Shape(kw["B"], kw["H"], kw["N"], kw["d"], topk=kw["topk"], group=kw["group"])
    assert m.mcs_workspace_bytes(s, m.MCS_OP_ANCHOR) == 0


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "free_sparse_attention_pddp_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), fn
                assert "mcs_oracle" not in text, fn


def test_packed_selection_size(lib):
    import free_sparse_attention_pddp_b200 as m

    s = m.Shape(1, 16, 65536, 64, topk=9830)
    assert m.mcs_meta_mask_bytes(s) == 16 * 512 * 2048 * 4
    s = m.Shape(2, 3, 1000, 128, topk=10)
    assert m.mcs_meta_mask_bytes(s) == 2 * 3 * 8 * 32 * 4
    assert m.mcs_meta_mask_bytes(m.Shape(1, 1, 1000, 128, topk=0)) == 0


def test_argument_errors_before_any_device_call(lib):
    """Host-side validation returns MCS_ERR_INVALID_ARG (1) before touching a GPU."""
    import ctypes as ct

    import free_sparse_attention_pddp_b200 as m

    s = m.Shape(1, 2, 1000, 128, topk=100)
    buf = (ct.c_uint8 * 4096)()
    p = ct.cast(buf, ct.c_void_p)
    # fast grouping: the Krylov step count must lie in [2, min(d, 64)] (one Lanczos cycle)
    for k in (0, 1, 65, 129):
        assert lib.mcs_group_fast(ct.byref(s), p, p, k, p, 4096, None) == 1
    # packed selection: null pointers, short status workspace
    assert lib.mcs_meta_pack(ct.byref(s), None, p, p, 4096, None) == 1
    assert lib.mcs_meta_unpack(ct.byref(s), p, None, p, 4096, None) == 1
    assert lib.mcs_meta_pack(ct.byref(s), p, p, p, 16, None) == 1
    # host-buffer reuse step: head chunks outside [1, min(H, 64)], missing buffers
    args = [ct.byref(s)] + [p] * 11
    assert lib.mcs_sparse_host(*args, 0, p, 4096, None, None, None) == 1
    assert lib.mcs_sparse_host(*args, 3, p, 4096, None, None, None) == 1
    nulls = [ct.byref(s), None] + [p] * 10
    assert lib.mcs_sparse_host(*nulls, 1, p, 4096, None, None, None) == 1
