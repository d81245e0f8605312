"""The C-ABI library loads and exports every entry point include/et.h
declares; host-side argument validation that needs no GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "et.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(et_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("et_build_graph", "et_run_splitk", "et_run_mlp", "et_run_moe", "et_sync_status", "et_get_trace",
              "et_destroy_graph", "et_status_str"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import event_driven_persistent_b200 as et
    lib = ctypes.CDLL(et.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert missing == []


def test_status_strings_and_null_checks():
    import event_driven_persistent_b200 as et
    assert et.et_status_str(0) == "ok"
    assert "timed out" in et.et_status_str(et.ET_ERR_TIMEOUT)
    lib = et._lib
    # null graph / null descriptor are rejected before any CUDA call
    assert lib.et_build_graph(None, None) == et.ET_ERR_INVALID
    assert lib.et_run_splitk(None, None, 1, None, None, None) == et.ET_ERR_INVALID
    assert lib.et_run_mlp(None, 1, None, None, None, None, None, None) == et.ET_ERR_INVALID
    assert lib.et_run_moe(None, 1, *([None] * 12)) == et.ET_ERR_INVALID
    assert lib.et_sync_status(None, None) == et.ET_ERR_INVALID
    # the allocation-free split-K rejects sizes beyond its maximum before any CUDA call
    assert lib.et_run_splitk_noalloc(None, 65537, None, None, None) == et.ET_ERR_INVALID
    assert lib.et_run_splitk_noalloc(None, 16, None, None, None) == et.ET_ERR_INVALID


def test_bad_descriptor_rejected():
    import event_driven_persistent_b200 as et
    with pytest.raises(et.EtError) as e:
        et.et_build_graph(et.ET_GRAPH_SPLITK, "static", 0)
    assert e.value.status == et.ET_ERR_INVALID
