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
    # O_dense fp32 + lse + queries in group order (bf16), all padded to 591
    # groups of 128, then a mass chunk of at most 2 GiB
    rows = 40 * 591 * 128
    fixed = rows * 128 * 4 + rows * 4 + rows * 128 * 2
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
