"""Python access to the CPU oracle of the DSA hot path (oracle/dsa_oracle.cpp).

TEST INFRASTRUCTURE ONLY. The tests, the smoke check and the benchmark's CPU
legs use it; the product path never does. Every number here is computed by the
plain C++ program (double precision, one query row at a time, rows spread over
std::threads); this module only converts numpy arrays and the workload dicts
of tests/case_utils.py into its arguments. It shares nothing with the CUDA
library and imports nothing from it.

The definitions it follows, and the readings taken where the DeepSeek-V3.2-Exp
pages are silent, are stated in oracle/dsa_oracle.cpp beside each function:
  * I[t,s] = sum_j w[t,j] * max(0, q_I[t,j] . k_I[s]) for s <= pos_t (jdon.com
    "DeepSeek-V3.2-Exp", lightning-indexer and matchmaking paragraphs);
  * the min(k, pos_t + 1) best positions under (score desc, position asc),
    ascending, -1 padded (same page, sparse-training and selection paragraphs);
  * per-head softmax attention over the selected latent rows, key = the whole
    row, value = its first Dv values (openi.cn "DeepSeek-V3.2", MLA-in-MQA item).
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build_oracle

_lib = None
_D = ctypes.POINTER(ctypes.c_double)
_F = ctypes.POINTER(ctypes.c_float)
_I = ctypes.POINTER(ctypes.c_int32)
_U8 = ctypes.POINTER(ctypes.c_uint8)
_U16 = ctypes.POINTER(ctypes.c_uint16)
_V = ctypes.c_void_p


class _Case(ctypes.Structure):
    _fields_ = [
        ("fp8", ctypes.c_int), ("B", ctypes.c_int), ("T", ctypes.c_int),
        ("H_I", ctypes.c_int), ("d_I", ctypes.c_int), ("H", ctypes.c_int), ("Dk", ctypes.c_int),
        ("Dv", ctypes.c_int), ("k", ctypes.c_int), ("softmax_scale", ctypes.c_double),
        ("seq_lens", _V), ("pos", _V), ("row_seq", _V),
        ("q_idx", _V), ("q_scale", _V), ("w", _V), ("q", _V),
        ("page_size", ctypes.c_int), ("n_max", ctypes.c_int),
        ("k_idx", _V), ("k_scale", _V), ("k_pages", _V), ("page_table", _V), ("max_pages", ctypes.c_int),
        ("kv", _V),
    ]


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build_oracle.build())
        ll, i, d = ctypes.c_longlong, ctypes.c_int, ctypes.c_double
        sig = {
            "oracle_hardware_threads": ([], i),
            "oracle_e4m3_value": ([ctypes.c_uint], d),
            "oracle_bf16_value": ([ctypes.c_uint], d),
            "oracle_decode_e4m3": ([_V, ll, _V], None),
            "oracle_decode_bf16": ([_V, ll, _V], None),
            "oracle_dequant": ([_V, ll, ll, _V, _V], None),
            "oracle_encode_e4m3": ([_V, ll, _V], None),
            "oracle_quantize_key_row": ([_V, i, _V, _V], None),
            "oracle_indexer_row": ([_V, _V, _V, ll, i, i, _V], None),
            "oracle_topk_row": ([_V, i, i, _V], None),
            "oracle_topk_rows": ([_V, ll, _V, i, i, _V, i], None),
            "oracle_sparse_attn_row": ([_V, _V, i, i, i, i, d, _V, _V], None),
            "oracle_seq_keys": ([ctypes.POINTER(_Case), i, _V, _V], None),
            "oracle_query_row": ([ctypes.POINTER(_Case), i, _V, _V, _V], None),
            "oracle_indexer_rows": ([ctypes.POINTER(_Case), _V, i, _V, ll, i], None),
            "oracle_attn_rows": ([ctypes.POINTER(_Case), _V, i, _V, _V, _V, i], None),
            "oracle_forward_rows": ([ctypes.POINTER(_Case), _V, i, _V, ll, _V, _V, _V, i], None),
            "oracle_cache_append": ([ctypes.POINTER(_Case), _V, _V, _V, _V, _V], None),
            "oracle_indexer_kl_row": ([_V, _V, i, i, i, d, _V, _V, _V], d),
            "oracle_attn_backward_row": ([_V, _V, i, i, i, i, d, _V, _V, _V], None),
            "oracle_attn_backward_seq": ([_V, _V, ll, _V, i, i, i, i, i, d, _V, _V, _V], None),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def threads() -> int:
    """Threads the oracle uses for many rows (the host's hardware threads)."""
    return int(lib().oracle_hardware_threads())


def _c(a, dtype):
    """C-contiguous array of `dtype` (no copy when it already is one) and its address."""
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(_V)


def _out(shape, dtype=np.float64):
    a = np.zeros(shape, dtype=dtype)
    return a, a.ctypes.data_as(_V)


# ---------------------------------------------------------------------------
# number formats

def e4m3_value(byte: int) -> float:
    """Value of one OCP FP8 E4M3 byte, from the format's bit fields."""
    return float(lib().oracle_e4m3_value(int(byte)))


def decode_e4m3(u8) -> np.ndarray:
    a, p = _c(u8, np.uint8)
    out, po = _out(a.shape)
    lib().oracle_decode_e4m3(p, a.size, po)
    return out


def decode_bf16(bits) -> np.ndarray:
    """bfloat16 bit patterns -> float64."""
    a, p = _c(np.asarray(bits).view(np.uint16), np.uint16)
    out, po = _out(a.shape)
    lib().oracle_decode_bf16(p, a.size, po)
    return out


def dequant(u8_rows, scale) -> np.ndarray:
    """x~ = s * dec(b) with one scale per leading row, in float64."""
    a, p = _c(u8_rows, np.uint8)
    s, ps = _c(np.asarray(scale).reshape(-1), np.float32)
    rows = s.size
    out, po = _out(a.shape)
    lib().oracle_dequant(p, rows, a.size // max(rows, 1), ps, po)
    return out


def encode_e4m3_rne(y) -> np.ndarray:
    """e4m3 byte of the value nearest to each y (ties to even), saturating; NaN -> 0x7F."""
    a, p = _c(y, np.float64)
    out, po = _out(a.shape, np.uint8)
    lib().oracle_encode_e4m3(p, a.size, po)
    return out


def quantize_key_row(x):
    """(e4m3 bytes, fp32 scale) of one indexer key row, in fp32 arithmetic."""
    a, p = _c(x, np.float32)
    codes, pc = _out(a.shape, np.uint8)
    sc = np.zeros(1, np.float32)
    lib().oracle_quantize_key_row(p, a.size, pc, sc.ctypes.data_as(_V))
    return codes, np.float32(sc[0])


# ---------------------------------------------------------------------------
# the stages on plain arrays

def indexer_row(q_t, w_t, keys) -> np.ndarray:
    """I[s] = sum_j w_t[j] * max(0, q_t[j] . keys[s]) for q_t [H_I, d_I], w_t [H_I], keys [n, d_I]."""
    q, pq = _c(q_t, np.float64)
    w, pw = _c(w_t, np.float64)
    k, pk = _c(keys, np.float64)
    H_I, d_I = q.shape
    n = k.shape[0] if k.ndim == 2 else 0
    out, po = _out(n)
    lib().oracle_indexer_row(pq, pw, pk, n, H_I, d_I, po)
    return out


def topk_row(scores, k: int) -> np.ndarray:
    """int32 [k]: the min(k, n) best positions (score desc, position asc; -0 == +0,
    NaN lowest) of a float32 row, ascending, -1 padded."""
    s, ps = _c(scores, np.float32)
    out, po = _out(int(k), np.int32)
    lib().oracle_topk_row(ps, s.size, int(k), po)
    return out


def topk_rows(scores, n, k: int, nthreads: int = 0) -> np.ndarray:
    """topk_row of every row r of a float32 [R, ld] array over its first n[r] entries."""
    s, ps = _c(scores, np.float32)
    nn, pn = _c(n, np.int32)
    R = nn.size
    out, po = _out((R, int(k)), np.int32)
    lib().oracle_topk_rows(ps, s.shape[1], pn, R, int(k), po, int(nthreads))
    return out


def sparse_attn_row(q_t, kv_rows, Dv: int, scale: float):
    """(o [H, Dv], lse [H]): softmax attention of q_t [H, Dk] over kv_rows [m, Dk]."""
    q, pq = _c(q_t, np.float64)
    r, pr = _c(kv_rows, np.float64)
    H, Dk = q.shape
    m = r.shape[0] if r.ndim == 2 else 0
    o, po = _out((H, int(Dv)))
    lse, pl = _out(H)
    lib().oracle_sparse_attn_row(pq, pr, m, H, Dk, int(Dv), float(scale), po, pl)
    return o, lse


# ---------------------------------------------------------------------------
# workload dicts (tests/case_utils.py) -> the oracle's case description

class _CaseRef:
    """A _Case and the arrays it points into (kept alive together)."""

    def __init__(self, case: dict):
        fp8 = bool(case["fp8"])
        keep = []

        def arr(x, dtype):
            if x is None:
                return None
            a = np.ascontiguousarray(x, dtype=dtype)
            keep.append(a)
            return a.ctypes.data_as(_V)

        c = _Case()
        c.fp8 = int(fp8)
        kv = case["kv"]
        seq = np.asarray(case["seq_lens"])
        pos = np.asarray(case.get("pos", np.zeros(0, np.int32)))
        c.B, c.T = int(seq.size), int(pos.size)
        c.d_I = int(case["d_I"])
        c.Dk = int(case.get("Dk", np.asarray(kv).shape[-1]))
        c.H_I, c.H, c.Dv, c.k = (int(case.get(x, 0)) for x in ("H_I", "H", "Dv", "k"))
        c.softmax_scale = float(case.get("softmax_scale", 1.0))
        c.seq_lens, c.pos = arr(seq, np.int32), arr(pos, np.int32)
        c.row_seq = arr(case.get("row_seq", np.zeros(0, np.int32)), np.int32)
        qt = np.uint8 if fp8 else np.float32
        c.q_idx = arr(case.get("q_idx"), qt)
        c.q_scale = arr(case.get("q_scale"), np.float32) if fp8 else None
        c.w = arr(case.get("w"), np.float32)
        q = case.get("q")
        c.q = arr(None if q is None else (np.asarray(q).view(np.uint16) if fp8 else q),
                  np.uint16 if fp8 else np.float32)
        c.page_size = int(case["page_size"])
        if c.page_size:
            pt = np.asarray(case["page_table"])
            c.page_table = arr(pt, np.int32)
            c.max_pages = int(pt.shape[1])
            c.k_pages = arr(case["k_pages"], np.uint8)
            c.n_max = 0
        else:
            c.k_idx = arr(case["k_idx"], np.uint8 if fp8 else np.float32)
            c.k_scale = arr(case.get("k_scale"), np.float32) if fp8 else None
            c.n_max = int(np.asarray(case["k_idx"]).shape[1])
        c.kv = arr(np.asarray(kv).view(np.uint16) if fp8 else kv, np.uint16 if fp8 else np.float32)
        self.c, self.keep = c, keep

    @property
    def ref(self):
        return ctypes.byref(self.c)


def seq_keys(case: dict, b: int):
    """Float64 indexer keys [len_b, d_I] and latent rows [len_b, Dk] of sequence b in
    position order (paged caches read through the page table)."""
    cr = _CaseRef(case)
    L = int(np.asarray(case["seq_lens"])[b])
    kI, pk = _out((L, cr.c.d_I))
    kv, pv = _out((L, cr.c.Dk))
    lib().oracle_seq_keys(cr.ref, int(b), pk, pv)
    return kI, kv


def query_row(case: dict, t: int):
    """Float64 (indexer query heads [H_I, d_I], weights [H_I], query heads [H, Dk]) of row t."""
    cr = _CaseRef(case)
    qI, p1 = _out((cr.c.H_I, cr.c.d_I))
    w, p2 = _out(cr.c.H_I)
    q, p3 = _out((cr.c.H, cr.c.Dk))
    lib().oracle_query_row(cr.ref, int(t), p1, p2, p3)
    return qI, w, q


def _rows(rows):
    r = np.ascontiguousarray(np.asarray(list(rows), dtype=np.int32))
    return r, r.ctypes.data_as(_V)


def indexer_rows(case: dict, rows, keys_cache=None, nthreads: int = 0):
    """Indexer scores of `rows` over their causal prefixes: {t: f64[pos+1]}."""
    cr = _CaseRef(case)
    r, pr = _rows(rows)
    pos = np.asarray(case["pos"])
    ld = int(max((int(pos[t]) + 1 for t in r), default=1))
    out, po = _out((r.size, ld))
    lib().oracle_indexer_rows(cr.ref, pr, r.size, po, ld, int(nthreads))
    return {int(t): out[i, :int(pos[t]) + 1] for i, t in enumerate(r)}


def attn_rows_on_indices(case: dict, rows, idx_rows, keys_cache=None, nthreads: int = 0):
    """Attention of `rows` recomputed on given selections (-1 = padding): {t: (o [H,Dv], lse [H])}."""
    cr = _CaseRef(case)
    r, pr = _rows(rows)
    k = cr.c.k
    ix = np.full((r.size, k), -1, np.int32)
    for i, x in enumerate(idx_rows):
        x = np.asarray(x, dtype=np.int32).reshape(-1)
        ix[i, :x.size] = x
    ix, pi = _c(ix, np.int32)
    o, po = _out((r.size, cr.c.H, cr.c.Dv))
    lse, pl = _out((r.size, cr.c.H))
    lib().oracle_attn_rows(cr.ref, pr, r.size, pi, po, pl, int(nthreads))
    return {int(t): (o[i], lse[i]) for i, t in enumerate(r)}


def forward_rows(case: dict, rows, keys_cache=None, nthreads: int = 0, want_scores: bool = True):
    """Indexer -> top-k (on the scores rounded to float32) -> attention for `rows`:
    {t: dict(scores=f64[pos+1], idx=int32[k], o=f64[H,Dv], lse=f64[H])}."""
    cr = _CaseRef(case)
    r, pr = _rows(rows)
    pos = np.asarray(case["pos"])
    ld = int(max((int(pos[t]) + 1 for t in r), default=1))
    sc, ps = _out((r.size, ld)) if want_scores else (None, None)
    idx, pi = _out((r.size, cr.c.k), np.int32)
    o, po = _out((r.size, cr.c.H, cr.c.Dv))
    lse, pl = _out((r.size, cr.c.H))
    lib().oracle_forward_rows(cr.ref, pr, r.size, ps, ld, pi, po, pl, int(nthreads))
    res = {}
    for i, t in enumerate(r):
        res[int(t)] = dict(scores=None if sc is None else sc[i, :int(pos[t]) + 1], idx=idx[i], o=o[i], lse=lse[i])
    return res


# ---------------------------------------------------------------------------
# cache write, indexer loss, attention backward

def cache_append(case: dict, k_new, kv_new_bits, k_pool, kv_pool_bits, k_scale=None):
    """Write row t's new indexer key (quantised per token) and latent row (bf16 bits)
    at its own position; returns updated copies (k_pool, kv_pool_bits, k_scale)."""
    kn, pk = _c(k_new, np.float32)
    kv_new = None if kv_new_bits is None else np.ascontiguousarray(np.asarray(kv_new_bits).view(np.uint16))
    k_pool = np.array(k_pool, dtype=np.uint8, copy=True, order="C")
    kv_pool_bits = np.array(np.asarray(kv_pool_bits).view(np.uint16), copy=True, order="C")
    k_scale = None if k_scale is None else np.array(k_scale, dtype=np.float32, copy=True, order="C")
    full = dict(fp8=True, seq_lens=np.zeros(1, np.int32), d_I=int(kn.shape[1]), kv=kv_pool_bits, k_pages=k_pool,
                k_idx=k_pool, k_scale=k_scale)
    full.update({x: case[x] for x in ("page_size", "row_seq", "pos", "page_table") if x in case})
    cr = _CaseRef(full)
    cr.c.T = int(kn.shape[0])
    lib().oracle_cache_append(cr.ref, pk, None if kv_new is None else kv_new.ctypes.data_as(_V),
                              k_pool.ctypes.data_as(_V), None if k_scale is None else k_scale.ctypes.data_as(_V),
                              kv_pool_bits.ctypes.data_as(_V))
    return k_pool, kv_pool_bits, k_scale


def indexer_kl_row(q_t, kv_rows, scale: float, scores):
    """(loss, target p [m], d loss / d scores [m]) for one row over its m selected rows."""
    q, pq = _c(q_t, np.float64)
    r, pr = _c(kv_rows, np.float64)
    s, ps = _c(scores, np.float64)
    H, Dk = q.shape
    m = s.size
    p, pp = _out(m)
    g, pg = _out(m)
    loss = lib().oracle_indexer_kl_row(pq, pr, m, H, Dk, float(scale), ps, pp, pg)
    return float(loss), p, g


def sparse_attn_backward_row(q_t, kv_rows, Dv: int, scale: float, dO):
    """(dq [H, Dk], dkv [m, Dk]): gradients of sum(dO * o) for one query row."""
    q, pq = _c(q_t, np.float64)
    r, pr = _c(kv_rows, np.float64)
    g, pg = _c(dO, np.float64)
    H, Dk = q.shape
    m = r.shape[0]
    dq, p1 = _out((H, Dk))
    dkv, p2 = _out((m, Dk))
    lib().oracle_attn_backward_row(pq, pr, m, H, Dk, int(Dv), float(scale), pg, p1, p2)
    return dq, dkv


def sparse_attn_backward_seq(q_rows, kv_seq, idx, Dv: int, scale: float, dO):
    """Backward over the query rows of one sequence: dq [R, H, Dk] and dkv [L, Dk]
    summed over every slot that selected each position."""
    q, pq = _c(q_rows, np.float64)
    kv, pk = _c(kv_seq, np.float64)
    ix, pi = _c(idx, np.int32)
    g, pg = _c(dO, np.float64)
    R, H, Dk = q.shape
    L = kv.shape[0]
    dq, p1 = _out((R, H, Dk))
    dkv, p2 = _out((L, Dk))
    lib().oracle_attn_backward_seq(pq, pk, L, pi, R, ix.shape[1], H, Dk, int(Dv), float(scale), pg, p1, p2)
    return dq, dkv
