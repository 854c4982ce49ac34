"""Python binding of libdsa.so (the C ABI in include/dsa.h).

Argument marshalling only: every stage runs in the library's CUDA kernels.
torch tensors supply device memory and the current CUDA stream. There is no
fallback: if the library is missing or a call fails, a DSAError is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsa.so")

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_CUDA, DSA_ERR_TIMEOUT, DSA_ERR_WORKSPACE, \
    DSA_ERR_DEVICE_CHECK, DSA_ERR_TOO_LARGE = range(8)
DSA_F32, DSA_BF16, DSA_E4M3 = 0, 1, 2
DSA_TOPK_AUTO, DSA_TOPK_SCORES, DSA_TOPK_FUSED = 0, 1, 2


class DSAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


class SeqLayout(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int),
        ("seq_lens", ctypes.c_void_p),
        ("cu_q", ctypes.c_void_p),
        ("page_size", ctypes.c_int),
        ("page_table", ctypes.c_void_p),
        ("max_pages", ctypes.c_int),
        ("num_pages", ctypes.c_int),
        ("n_max", ctypes.c_int),
    ]


class ForwardArgs(ctypes.Structure):
    _fields_ = [
        ("q_idx", ctypes.c_void_p), ("q_scale", ctypes.c_void_p),
        ("k_idx", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
        ("idx_dt", ctypes.c_int), ("w", ctypes.c_void_p), ("H_I", ctypes.c_int), ("d_I", ctypes.c_int),
        ("q", ctypes.c_void_p), ("kv", ctypes.c_void_p), ("attn_dt", ctypes.c_int),
        ("H", ctypes.c_int), ("Dk", ctypes.c_int), ("Dv", ctypes.c_int), ("softmax_scale", ctypes.c_float),
        ("k", ctypes.c_int), ("T", ctypes.c_int),
        ("lay", SeqLayout),
        ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p), ("idx_out", ctypes.c_void_p),
        ("topk_path", ctypes.c_int),
    ]


_lib = None

EXPORTS = ("dsa_indexer_scores", "dsa_topk", "dsa_sparse_mqa_attn_workspace_size", "dsa_sparse_mqa_attn",
           "dsa_forward_workspace_size", "dsa_forward", "dsa_get_device_error", "dsa_set_wait_limit_ns",
           "dsa_status_string", "dsa_version", "dsa_sparse_mqa_attn_noalloc", "dsa_get_device_error_site",
           "dsa_cache_append", "dsa_indexer_kl", "dsa_sparse_mqa_attn_backward",
           "dsa_sparse_mqa_attn_backward_workspace_size", "dsa_topk_from_candidates", "dsa_indexer_candidates")


def lib() -> ctypes.CDLL:
    """Load libdsa.so from the package directory (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m sparse_long_context_04_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, ll, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t
        L.dsa_indexer_scores.argtypes = [vp, vp, vp, vp, i, vp, i, i, i, ctypes.POINTER(SeqLayout), vp, ll, vp]
        L.dsa_topk.argtypes = [vp, ll, i, i, ctypes.POINTER(SeqLayout), vp, vp]
        L.dsa_topk_from_candidates.argtypes = [vp, vp, vp, ll, vp, i, i, ctypes.POINTER(SeqLayout), vp, vp]
        L.dsa_topk_from_candidates.restype = i
        L.dsa_indexer_candidates.argtypes = [vp, vp, vp, vp, i, vp, i, i, i, ctypes.POINTER(SeqLayout), i, vp, vp,
                                             vp, vp, ll, vp]
        L.dsa_indexer_candidates.restype = i
        L.dsa_sparse_mqa_attn_workspace_size.argtypes = [i, i, i, i, i]
        L.dsa_sparse_mqa_attn_workspace_size.restype = sz
        L.dsa_sparse_mqa_attn.argtypes = [vp, vp, i, i, i, i, i, ctypes.c_float, vp, i, ctypes.POINTER(SeqLayout),
                                          vp, vp, vp, sz, vp]
        L.dsa_sparse_mqa_attn_noalloc.argtypes = [vp, vp, i, i, i, i, i, ctypes.c_float, vp, i,
                                                  ctypes.POINTER(SeqLayout), vp, vp, vp]
        L.dsa_sparse_mqa_attn_noalloc.restype = i
        L.dsa_cache_append.argtypes = [vp, i, vp, i, i, i, ctypes.POINTER(SeqLayout), vp, vp, vp, vp]
        L.dsa_cache_append.restype = i
        L.dsa_indexer_kl.argtypes = [vp, vp, i, i, i, i, ctypes.c_float, vp, i, ctypes.POINTER(SeqLayout), vp, vp,
                                     ll, vp, vp, vp]
        L.dsa_indexer_kl.restype = i
        L.dsa_sparse_mqa_attn_backward_workspace_size.argtypes = [i]
        L.dsa_sparse_mqa_attn_backward_workspace_size.restype = sz
        L.dsa_sparse_mqa_attn_backward.argtypes = [vp, vp, i, i, i, i, i, ctypes.c_float, vp, i,
                                                   ctypes.POINTER(SeqLayout), vp, vp, vp, vp, vp, vp, sz, vp]
        L.dsa_sparse_mqa_attn_backward.restype = i
        L.dsa_forward_workspace_size.argtypes = [ctypes.POINTER(ForwardArgs)]
        L.dsa_forward_workspace_size.restype = sz
        L.dsa_forward.argtypes = [ctypes.POINTER(ForwardArgs), vp, sz, vp]
        L.dsa_get_device_error.argtypes = [vp]
        L.dsa_get_device_error_site.argtypes = [vp, ctypes.POINTER(ctypes.c_uint)]
        L.dsa_get_device_error_site.restype = i
        L.dsa_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
        L.dsa_status_string.argtypes = [i]
        L.dsa_status_string.restype = ctypes.c_char_p
        L.dsa_version.restype = i
        for name in ("dsa_indexer_scores", "dsa_topk", "dsa_sparse_mqa_attn", "dsa_forward",
                     "dsa_get_device_error", "dsa_set_wait_limit_ns"):
            getattr(L, name).restype = i
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().dsa_status_string(int(s)).decode()


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(s: int, what: str):
    if s != DSA_OK:
        raise DSAError(s, what)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return DSA_F32
    if t.dtype == torch.bfloat16:
        return DSA_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return DSA_E4M3
    raise TypeError(f"unsupported dtype {t.dtype}")


class Layout:
    """A dsa_seq_layout plus references to the device tensors it points into."""

    def __init__(self, seq_lens, n_max, cu_q=None, page_table=None, page_size=0, num_pages=0):
        self.seq_lens, self.cu_q, self.page_table = seq_lens, cu_q, page_table
        self.c = SeqLayout(
            batch=int(seq_lens.numel()), seq_lens=seq_lens.data_ptr(),
            cu_q=None if cu_q is None else cu_q.data_ptr(), page_size=int(page_size),
            page_table=None if page_table is None else page_table.data_ptr(),
            max_pages=0 if page_table is None else int(page_table.shape[1]),
            num_pages=int(num_pages), n_max=int(n_max))

    @property
    def capacity(self) -> int:
        return self.c.max_pages * self.c.page_size if self.c.page_size else self.c.n_max


def dsa_indexer_scores(q_idx, q_scale, k_idx, k_scale, w, layout: Layout, scores, T=None, stream=None):
    T = q_idx.shape[0] if T is None else T
    H_I, d_I = int(q_idx.shape[1]), int(q_idx.shape[2])
    s = lib().dsa_indexer_scores(_p(q_idx), _p(q_scale), _p(k_idx), _p(k_scale), _dt(q_idx), _p(w), int(T), H_I,
                                 d_I, ctypes.byref(layout.c), _p(scores), int(scores.stride(0)), _stream(stream))
    _check(s, "dsa_indexer_scores")


def dsa_topk(scores, k, layout: Layout, idx, T=None, stream=None):
    T = scores.shape[0] if T is None else T
    s = lib().dsa_topk(_p(scores), int(scores.stride(0)), int(T), int(k), ctypes.byref(layout.c), _p(idx),
                       _stream(stream))
    _check(s, "dsa_topk")


def dsa_indexer_candidates(q_idx, q_scale, k_idx, k_scale, w, layout: Layout, k, hist, cand_score, cand_pos,
                           cand_count, stream=None):
    """Fused indexer -> top-k, producer half (decode rows): each row's candidates
    and their 12-bit order-key histogram, instead of its scores (see
    include/dsa.h). cand_score/cand_pos [T][cap] with cap >= the cache capacity."""
    T = int(q_idx.shape[0])
    H_I, d_I = int(q_idx.shape[1]), int(q_idx.shape[2])
    cap = int(cand_score.shape[1])
    s = lib().dsa_indexer_candidates(_p(q_idx), _p(q_scale), _p(k_idx), _p(k_scale), _dt(q_idx), _p(w), T, H_I, d_I,
                                     ctypes.byref(layout.c), int(k), _p(hist), _p(cand_score), _p(cand_pos),
                                     _p(cand_count), cap, _stream(stream))
    _check(s, "dsa_indexer_candidates")


def dsa_topk_from_candidates(score, pos, count, hist, k, layout: Layout, idx, stream=None):
    """Top-k of each row from its candidate list and complete 12-bit histogram
    (see include/dsa.h): score/pos [T][cap], count [T], hist [T][4096]."""
    T, cap = (int(x) for x in score.shape)
    s = lib().dsa_topk_from_candidates(_p(score), _p(pos), _p(count), cap, _p(hist), T, int(k),
                                       ctypes.byref(layout.c), _p(idx), _stream(stream))
    _check(s, "dsa_topk_from_candidates")


def dsa_sparse_mqa_attn_workspace_size(T, H, Dv, k, dtype) -> int:
    return int(lib().dsa_sparse_mqa_attn_workspace_size(int(T), int(H), int(Dv), int(k), _dt(dtype)))


def dsa_sparse_mqa_attn(q, kv, idx, layout: Layout, out, lse, softmax_scale, workspace=None, stream=None):
    T, H, Dk = (int(x) for x in q.shape)
    Dv = int(out.shape[2])
    k = int(idx.shape[1])
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    s = lib().dsa_sparse_mqa_attn(_p(q), _p(kv), _dt(q), T, H, Dk, Dv, float(softmax_scale), _p(idx), k,
                                  ctypes.byref(layout.c), _p(out), _p(lse), _p(workspace), ws_bytes,
                                  _stream(stream))
    _check(s, "dsa_sparse_mqa_attn")


def dsa_cache_append(k_new, kv_new, layout: Layout, k_cache, kv_cache, k_scale=None, stream=None):
    """Write each query row's new indexer key (quantised to e4m3 with a per-token
    scale) and latent row at the row's own position (see include/dsa.h)."""
    T, d_I = (int(x) for x in k_new.shape)
    Dk = 0 if kv_new is None else int(kv_new.shape[1])
    s = lib().dsa_cache_append(_p(k_new), _dt(k_new), _p(kv_new), T, d_I, Dk, ctypes.byref(layout.c),
                               _p(k_cache), _p(k_scale), _p(kv_cache), _stream(stream))
    _check(s, "dsa_cache_append")


def dsa_indexer_kl(q, kv, idx, layout: Layout, lse, scores, loss, softmax_scale, grad=None, stream=None):
    """Indexer loss on the selected set: KL(heads' mean attention || softmax of the
    indexer scores) per row into `loss`, and its gradient with respect to the
    selected scores into `grad` (see include/dsa.h)."""
    T, H, Dk = (int(x) for x in q.shape)
    s = lib().dsa_indexer_kl(_p(q), _p(kv), _dt(q), T, H, Dk, float(softmax_scale), _p(idx), int(idx.shape[1]),
                             ctypes.byref(layout.c), _p(lse), _p(scores), int(scores.stride(0)), _p(loss), _p(grad),
                             _stream(stream))
    _check(s, "dsa_indexer_kl")


def dsa_sparse_mqa_attn_backward_workspace_size(T) -> int:
    return int(lib().dsa_sparse_mqa_attn_backward_workspace_size(int(T)))


def dsa_sparse_mqa_attn_backward(q, kv, idx, layout: Layout, out, dout, lse, dq, dkv, softmax_scale, workspace,
                                 stream=None):
    """Gradients of the sparse attention output with respect to q and the selected
    latent rows, accumulated into dq and dkv (fp32; see include/dsa.h)."""
    T, H, Dk = (int(x) for x in q.shape)
    ws_bytes = workspace.numel() * workspace.element_size()
    s = lib().dsa_sparse_mqa_attn_backward(_p(q), _p(kv), _dt(q), T, H, Dk, int(out.shape[2]),
                                           float(softmax_scale), _p(idx), int(idx.shape[1]), ctypes.byref(layout.c),
                                           _p(out), _p(dout), _p(lse), _p(dq), _p(dkv), _p(workspace), ws_bytes,
                                           _stream(stream))
    _check(s, "dsa_sparse_mqa_attn_backward")


def dsa_sparse_mqa_attn_noalloc(q, kv, idx, layout: Layout, out, lse, softmax_scale, stream=None):
    """Stage 3 with the library's built-in scratch instead of a caller workspace
    (for callers that may not allocate device memory; see include/dsa.h)."""
    T, H, Dk = (int(x) for x in q.shape)
    s = lib().dsa_sparse_mqa_attn_noalloc(_p(q), _p(kv), _dt(q), T, H, Dk, int(out.shape[2]),
                                          float(softmax_scale), _p(idx), int(idx.shape[1]),
                                          ctypes.byref(layout.c), _p(out), _p(lse), _stream(stream))
    _check(s, "dsa_sparse_mqa_attn_noalloc")


def forward_args(q_idx, q_scale, k_idx, k_scale, w, q, kv, k, softmax_scale, layout: Layout, out, lse=None,
                 idx_out=None, topk_path=DSA_TOPK_AUTO) -> ForwardArgs:
    a = ForwardArgs()
    a.q_idx, a.q_scale, a.k_idx, a.k_scale = (t.data_ptr() if t is not None else None
                                              for t in (q_idx, q_scale, k_idx, k_scale))
    a.idx_dt = _dt(q_idx)
    a.w = w.data_ptr()
    a.H_I, a.d_I = int(q_idx.shape[1]), int(q_idx.shape[2])
    a.q, a.kv = q.data_ptr(), kv.data_ptr()
    a.attn_dt = _dt(q)
    a.H, a.Dk = int(q.shape[1]), int(q.shape[2])
    a.Dv = int(out.shape[2])
    a.softmax_scale = float(softmax_scale)
    a.k = int(k)
    a.T = int(q.shape[0])
    a.lay = layout.c
    a.out = out.data_ptr()
    a.lse = None if lse is None else lse.data_ptr()
    a.idx_out = None if idx_out is None else idx_out.data_ptr()
    a.topk_path = int(topk_path)
    return a


def dsa_forward_workspace_size(args: ForwardArgs) -> int:
    return int(lib().dsa_forward_workspace_size(ctypes.byref(args)))


def dsa_forward(args: ForwardArgs, workspace, stream=None):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    s = lib().dsa_forward(ctypes.byref(args), _p(workspace), ws_bytes, _stream(stream))
    _check(s, "dsa_forward")


def dsa_get_device_error(stream=None) -> int:
    return int(lib().dsa_get_device_error(_stream(stream)))


def dsa_get_device_error_site(stream=None):
    """(status, site code of the first failing device check or wait)."""
    site = ctypes.c_uint(0)
    st = int(lib().dsa_get_device_error_site(_stream(stream), ctypes.byref(site)))
    return st, int(site.value)


def dsa_set_wait_limit_ns(ns: int):
    _check(lib().dsa_set_wait_limit_ns(int(ns)), "dsa_set_wait_limit_ns")
