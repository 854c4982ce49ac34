"""The C ABI library loads on a machine without a GPU, exports every entry point
include/dsa.h declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

from sparse_long_context_04_b200 import dsa as D

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "dsa.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(D.LIB_PATH):
        from sparse_long_context_04_b200 import build
        build.build()
    return D.lib()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(D.EXPORTS) <= set(names)


def test_status_strings_and_version(lib):
    assert lib.dsa_version() >= 100
    assert D.status_string(D.DSA_OK) == "ok"
    assert "workspace" in D.status_string(D.DSA_ERR_WORKSPACE)
    assert D.status_string(99) == "unknown status"


def test_host_rejects_bad_arguments_without_gpu(lib):
    vp = ctypes.c_void_p
    # no layout
    assert lib.dsa_topk(vp(16), 4, 1, 8, None, vp(16), None) == D.DSA_ERR_INVALID_ARG
    assert lib.dsa_indexer_scores(vp(16), vp(16), vp(16), vp(16), D.DSA_E4M3, vp(16), 1, 64, 128, None, vp(16),
                                  128, None) == D.DSA_ERR_INVALID_ARG
    assert lib.dsa_forward(None, None, 0, None) == D.DSA_ERR_INVALID_ARG
    # decode layout whose row count differs from the batch
    lay = D.SeqLayout(batch=2, seq_lens=16, cu_q=None, page_size=0, page_table=None, max_pages=0,
                      num_pages=0, n_max=64)
    assert lib.dsa_topk(vp(16), 64, 3, 8, ctypes.byref(lay), vp(16), None) == D.DSA_ERR_INVALID_ARG
    # page size other than 0 or 64
    lay.page_size = 32
    assert lib.dsa_topk(vp(16), 64, 2, 8, ctypes.byref(lay), vp(16), None) == D.DSA_ERR_UNSUPPORTED
    # paged layout without a page table
    lay.page_size = 64
    assert lib.dsa_topk(vp(16), 64, 2, 8, ctypes.byref(lay), vp(16), None) == D.DSA_ERR_INVALID_ARG
    assert lib.dsa_set_wait_limit_ns(0) == D.DSA_ERR_INVALID_ARG
