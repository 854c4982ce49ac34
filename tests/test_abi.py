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


def _decode_layout(batch=2, page_size=0):
    return D.SeqLayout(batch=batch, seq_lens=16, cu_q=None, page_size=page_size,
                       page_table=32 if page_size else None, max_pages=4 if page_size else 0,
                       num_pages=8 if page_size else 0, n_max=256)


def test_cache_append_rejects_bad_arguments_without_gpu(lib):
    vp = ctypes.c_void_p
    A = 4096  # a 16-byte-aligned stand-in address; no call below reaches the device
    paged, contig = _decode_layout(page_size=64), _decode_layout()
    ok_paged = dict(k_new=vp(A), k_dt=D.DSA_F32, kv_new=vp(A), T=2, d_I=128, Dk=576, k_cache=vp(A),
                    k_scale=None, kv_cache=vp(A))

    def call(lay, **kw):
        a = dict(ok_paged, **kw)
        return lib.dsa_cache_append(a["k_new"], a["k_dt"], a["kv_new"], a["T"], a["d_I"], a["Dk"],
                                    ctypes.byref(lay), a["k_cache"], a["k_scale"], a["kv_cache"], None)

    assert call(paged, k_new=None) == D.DSA_ERR_INVALID_ARG
    assert call(paged, k_dt=D.DSA_E4M3) == D.DSA_ERR_UNSUPPORTED
    assert call(paged, d_I=64) == D.DSA_ERR_UNSUPPORTED
    assert call(paged, k_new=vp(A + 4)) == D.DSA_ERR_INVALID_ARG          # fp32 rows need 16-byte alignment
    assert call(paged, k_scale=vp(A)) == D.DSA_ERR_INVALID_ARG           # paged pools keep scales in the pages
    assert call(contig) == D.DSA_ERR_INVALID_ARG                          # contiguous caches need k_scale
    assert call(paged, Dk=580) == D.DSA_ERR_INVALID_ARG                   # latent rows in 16-byte pieces
    assert call(paged, kv_cache=None) == D.DSA_ERR_INVALID_ARG
    assert call(paged, T=3) == D.DSA_ERR_INVALID_ARG                      # decode: one row per sequence
    # nothing to do: accepted without touching the device
    cu = _decode_layout()
    cu.cu_q = A
    assert call(cu, T=0, k_scale=vp(A)) == D.DSA_OK


def test_attention_rejects_shapes_without_a_kernel_without_gpu(lib):
    vp = ctypes.c_void_p
    A = 4096
    lay = _decode_layout()

    def attn(dt=D.DSA_BF16, H=128, Dk=576, Dv=512, k=2048, q=A):
        return lib.dsa_sparse_mqa_attn(vp(q), vp(A), dt, 2, H, Dk, Dv, ctypes.c_float(0.1), vp(A), k,
                                       ctypes.byref(lay), vp(A), vp(A), vp(A), ctypes.c_size_t(1 << 20), None)

    assert attn(H=64) == D.DSA_ERR_UNSUPPORTED
    assert attn(Dk=512, Dv=512) == D.DSA_ERR_UNSUPPORTED
    assert attn(k=16385) == D.DSA_ERR_UNSUPPORTED
    assert attn(q=A + 2) == D.DSA_ERR_INVALID_ARG
    assert attn(Dv=600) == D.DSA_ERR_INVALID_ARG                          # the value is a prefix of the key row
    # the built-in-scratch entry point takes bf16 only
    assert lib.dsa_sparse_mqa_attn_noalloc(vp(A), vp(A), D.DSA_F32, 2, 8, 64, 32, ctypes.c_float(0.1), vp(A), 64,
                                           ctypes.byref(lay), vp(A), vp(A), None) == D.DSA_ERR_UNSUPPORTED


def test_indexer_kl_rejects_bad_arguments_without_gpu(lib):
    vp = ctypes.c_void_p
    A = 4096
    lay = _decode_layout()          # contiguous, n_max 256

    def kl(dt=D.DSA_BF16, H=128, Dk=576, k=2048, ld=256, q=A, kv=A, loss=A, grad=A, lse=A, T=2):
        return lib.dsa_indexer_kl(vp(q), vp(kv), dt, T, H, Dk, ctypes.c_float(0.1), vp(A), k, ctypes.byref(lay),
                                  vp(lse), vp(A), ld, vp(loss), vp(grad), None)

    assert kl(loss=None) == D.DSA_ERR_INVALID_ARG
    assert kl(lse=None) == D.DSA_ERR_INVALID_ARG
    assert kl(ld=252) == D.DSA_ERR_INVALID_ARG                            # score rows shorter than the cache
    assert kl(dt=D.DSA_F32) == D.DSA_ERR_UNSUPPORTED
    assert kl(H=64) == D.DSA_ERR_UNSUPPORTED
    assert kl(k=16385) == D.DSA_ERR_UNSUPPORTED
    assert kl(kv=A + 8) == D.DSA_ERR_INVALID_ARG                          # latent rows in 16-byte pieces
    assert kl(q=A + 4) == D.DSA_ERR_INVALID_ARG                           # the query block is read by TMA
    assert kl(grad=A + 2) == D.DSA_ERR_INVALID_ARG
    assert kl(T=3) == D.DSA_ERR_INVALID_ARG                               # decode: one row per sequence


def test_attention_backward_rejects_bad_arguments_without_gpu(lib):
    vp = ctypes.c_void_p
    A = 4096
    lay = _decode_layout()

    def bwd(dt=D.DSA_BF16, H=128, Dk=576, Dv=512, k=2048, dq=A, lse=A, ws=A, ws_bytes=1 << 20, T=2):
        return lib.dsa_sparse_mqa_attn_backward(vp(A), vp(A), dt, T, H, Dk, Dv, ctypes.c_float(0.1), vp(A), k,
                                                ctypes.byref(lay), vp(A), vp(A), vp(lse), vp(dq), vp(A), vp(ws),
                                                ctypes.c_size_t(ws_bytes), None)

    assert bwd(dq=None) == D.DSA_ERR_INVALID_ARG
    assert bwd(dt=D.DSA_F32) == D.DSA_ERR_UNSUPPORTED
    assert bwd(H=64) == D.DSA_ERR_UNSUPPORTED
    assert bwd(k=16385) == D.DSA_ERR_UNSUPPORTED
    assert bwd(Dv=600) == D.DSA_ERR_INVALID_ARG                           # the value is a prefix of the row
    assert bwd(dq=A + 4) == D.DSA_ERR_INVALID_ARG                         # fp32 rows added 16 bytes at a time
    assert bwd(lse=A + 2) == D.DSA_ERR_INVALID_ARG
    assert bwd(ws=None) == D.DSA_ERR_WORKSPACE
    assert bwd(ws_bytes=512) == D.DSA_ERR_WORKSPACE                       # two rows need 1 KiB of dO . o
    assert bwd(ws=A + 128) == D.DSA_ERR_WORKSPACE
    assert lib.dsa_sparse_mqa_attn_backward_workspace_size(2) == 1024
    assert lib.dsa_sparse_mqa_attn_backward_workspace_size(0) == 0


def test_topk_from_candidates_rejects_bad_arguments_without_gpu(lib):
    vp = ctypes.c_void_p
    A = 4096
    lay = _decode_layout()

    def call(score=A, count=A, hist=A, k=2048, cap=256, T=2, n_max=256):
        lay.n_max = n_max
        return lib.dsa_topk_from_candidates(vp(score), vp(A), vp(count), cap, vp(hist), T, k, ctypes.byref(lay),
                                            vp(A), None)

    assert call(hist=None) == D.DSA_ERR_INVALID_ARG
    assert call(count=None) == D.DSA_ERR_INVALID_ARG
    assert call(k=0) == D.DSA_ERR_INVALID_ARG
    assert call(cap=0) == D.DSA_ERR_INVALID_ARG
    assert call(T=3) == D.DSA_ERR_INVALID_ARG                             # decode: one row per sequence
    assert call(n_max=262145) == D.DSA_ERR_UNSUPPORTED                    # rows up to 262144 keys
