"""A second, independent statement of the DSA hot path in numpy (float64).

TEST INFRASTRUCTURE ONLY, and not the oracle: the oracle is the plain C++
program in oracle/dsa_oracle.cpp. This numpy restatement was written first and
is kept as one more pin of the oracle: `tests/test_oracle_cpp.py` checks that
the two agree on the pin cases. Only the tests import it. It shares no code with
the C++ oracle or with the CUDA library.

Sources (the DeepSeek-V3.2-Exp pages; none prints an equation, so each stage is
written from the words):
  [jdon-indexer]   jdon.com "DeepSeek-V3.2-Exp", paragraph introducing the
                   lightning indexer: light enough for FP8, very few heads, scores
                   each query token against each earlier token with a weighted
                   sum of ReLU-activated dot products.
  [jdon-matchmake] same page, the "matchmaking" analogy paragraph: ReLU applied to
                   the q_I/k_I meeting score, w_I as the weight, the highest scores
                   go into the top-k set; main attention cost O(L^2) -> O(L*k).
  [jdon-sparse]    same page, sparse-training paragraph: each query keeps only the
                   2048 (K = 2048) highest-scoring earlier tokens.
  [jdon-select]    same page, fine-grained selection paragraph: only the k chosen
                   key/value entries take part; the output hidden state is u_t.
  [jdon-causal]    same page, opening paragraph on cost: every token otherwise
                   attends to all tokens before it (O(L^2)).
  [openi-mla]      openi.cn "DeepSeek-V3.2", technical section, items on the
                   lightning indexer (scores between the query token and earlier
                   tokens), token selection (top-k value entries) and MLA in MQA
                   mode (one value entry shared by many queries).
  [mundobytes-run] mundobytes.com run guide: the serving command uses page size 64.
  [mundobytes-kernels] same page, open-kernels paragraph: the indexer kernels are
                   published in a paged version.

Readings taken where the pages are silent:
  * I[t,s] = sum_j w[t,j] * max(0, q_I[t,j] . k_I[s]), ReLU per head before the
    weighted sum; the FP8 per-token scales multiply the dequantised vectors.
  * causal set s <= pos_t, inclusive of the query's own position.
  * top-k order: score descending, then index ascending; -0 == +0; NaN lowest;
    emitted in ascending index order, padded with -1 when pos_t + 1 < k.
  * attention: key = full latent row (Dk dims), value = its first Dv dims, one
    row shared by all heads; plain softmax with a caller-given scale, no sink.
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# number formats


def e4m3_value(byte: int) -> float:
    """Value of one OCP FP8 E4M3 ("e4m3fn") byte, from the format definition:
    1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent 0 is
    subnormal (m/8 * 2^-6); S.1111.111 is NaN; there is no infinity."""
    s = (byte >> 7) & 1
    e = (byte >> 3) & 0xF
    m = byte & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        mag = (m / 8.0) * 2.0 ** (-6)
    else:
        mag = (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return -mag if s else mag


E4M3_TABLE = np.array([e4m3_value(b) for b in range(256)], dtype=np.float64)


def decode_e4m3(u8: np.ndarray) -> np.ndarray:
    return E4M3_TABLE[np.asarray(u8, dtype=np.uint8)]


def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float64 (bf16 is the top half of an IEEE binary32)."""
    b = np.asarray(bits).view(np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def dequant(u8_rows: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """x~ = s * dec(b) with one scale per leading row, in float64."""
    x = decode_e4m3(u8_rows)
    s = np.asarray(scale, dtype=np.float64).reshape((-1,) + (1,) * (x.ndim - 1))
    return x * s


# ---------------------------------------------------------------------------
# stage 1: lightning indexer   [jdon-indexer], [jdon-matchmake], [openi-mla]


def indexer_row(q_t: np.ndarray, w_t: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """Scores of one query token against `keys` (its causal prefix).

    q_t  [H_I, d_I] float64: the token's indexer query heads (dequantised)
    w_t  [H_I]      float64: the token's per-head weights
    keys [n, d_I]   float64: indexer keys of positions 0..n-1 (dequantised)
    returns I[s] = sum_j w_t[j] * max(0, q_t[j] . keys[s]),  s = 0..n-1
    """
    dots = keys @ q_t.T                      # [n, H_I]: q_I[t,j] . k_I[s]
    return np.maximum(dots, 0.0) @ w_t       # ReLU per head, then the weighted sum


# ---------------------------------------------------------------------------
# stage 2: fine-grained token selection   [jdon-sparse], [jdon-select], [openi-mla]


def topk_row(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices kept for one query row.

    scores: float32 [n] — the row's scores over its causal prefix s = 0..n-1.
    Returns int32 [k]: the m = min(k, n) indices that come first under the order
    (score descending, index ascending), listed in ascending index order and
    padded with -1. -0.0 and +0.0 compare equal; NaN ranks below every number.
    """
    v = np.asarray(scores, dtype=np.float32).astype(np.float64)
    n = v.shape[0]
    m = min(k, n)
    idx = np.arange(n)
    # primary key: -v ascending (NaN sorts last); secondary: index ascending
    order = np.lexsort((idx, -v))
    chosen = np.sort(order[:m])
    out = np.full(k, -1, dtype=np.int32)
    out[:m] = chosen
    return out


# ---------------------------------------------------------------------------
# stage 3: sparse MQA attention over the latent rows   [jdon-select], [openi-mla]


def sparse_attn_row(q_t: np.ndarray, kv_rows: np.ndarray, Dv: int, scale: float):
    """Attention of one query token over its selected latent rows.

    q_t     [H, Dk] float64: the token's query heads
    kv_rows [m, Dk] float64: the selected rows (key = whole row, value = first Dv dims)
    returns (o [H, Dv], lse [H]) with z = scale * q.k, o = softmax(z) @ v,
    lse = log sum exp z (natural log). Two-pass softmax.
    """
    z = scale * (q_t @ kv_rows.T)                   # [H, m]
    zmax = z.max(axis=1, keepdims=True)
    p = np.exp(z - zmax)
    Z = p.sum(axis=1, keepdims=True)
    o = (p @ kv_rows[:, :Dv]) / Z
    lse = zmax[:, 0] + np.log(Z[:, 0])
    return o, lse


def dense_causal_mqa_online(q_t: np.ndarray, kv_prefix: np.ndarray, Dv: int, scale: float):
    """Dense causal MQA for one token, written as a one-key-at-a-time online
    softmax (a different algorithm from `sparse_attn_row`). Used to pin the
    invariant that DSA with k >= L equals dense causal attention."""
    H = q_t.shape[0]
    m = np.full(H, -np.inf)
    l = np.zeros(H)
    acc = np.zeros((H, Dv))
    for s in range(kv_prefix.shape[0]):
        z = scale * (q_t @ kv_prefix[s])
        m_new = np.maximum(m, z)
        a = np.exp(m - m_new)
        b = np.exp(z - m_new)
        l = l * a + b
        acc = acc * a[:, None] + b[:, None] * kv_prefix[s, :Dv][None, :]
        m = m_new
    return acc / l[:, None], m + np.log(l)


# ---------------------------------------------------------------------------
# logical views of the key caches (contiguous or paged)  [mundobytes-run]


def seq_keys(case: dict, b: int):
    """Float64 indexer keys [len_b, d_I] and latent rows [len_b, Dk] of sequence b,
    in logical position order. A paged cache maps position s to page
    page_table[b, s // P], slot s % P; an indexer page holds P key rows of d_I
    bytes followed by P little-endian float32 scales."""
    L = int(case["seq_lens"][b])
    fp8 = case["fp8"]
    P = case["page_size"]
    if P == 0:
        if fp8:
            kI = dequant(case["k_idx"][b, :L], case["k_scale"][b, :L])
            kv = decode_bf16(case["kv"][b, :L])
        else:
            kI = np.asarray(case["k_idx"][b, :L], dtype=np.float64)
            kv = np.asarray(case["kv"][b, :L], dtype=np.float64)
        return kI, kv
    d_I = case["d_I"]
    pos = np.arange(L)
    page = case["page_table"][b, pos // P].astype(np.int64)
    slot = pos % P
    pages = case["k_pages"]
    kbytes = pages[page[:, None], slot[:, None] * d_I + np.arange(d_I)[None, :]]
    sbytes = pages[page[:, None], P * d_I + slot[:, None] * 4 + np.arange(4)[None, :]]
    scale = np.ascontiguousarray(sbytes).view("<f4").reshape(L)
    kI = dequant(kbytes, scale)
    kv = decode_bf16(case["kv"][page, slot])
    return kI, kv


def query_row(case: dict, t: int):
    """Float64 (indexer query heads [H_I, d_I], weights [H_I], query heads [H, Dk]) of row t."""
    if case["fp8"]:
        qI = dequant(case["q_idx"][t][None], case["q_scale"][t:t + 1])[0]
        q = decode_bf16(case["q"][t])
    else:
        qI = np.asarray(case["q_idx"][t], dtype=np.float64)
        q = np.asarray(case["q"][t], dtype=np.float64)
    w = np.asarray(case["w"][t], dtype=np.float64)
    return qI, w, q


# ---------------------------------------------------------------------------
# whole path for chosen rows


def forward_rows(case: dict, rows, keys_cache=None):
    """Indexer -> top-k -> attention for query rows `rows` of `case`.

    Returns {t: dict(scores=f64[pos+1], idx=int32[k], o=f64[H,Dv], lse=f64[H])}.
    The selection runs on the oracle's own scores rounded to float32.
    """
    keys_cache = {} if keys_cache is None else keys_cache
    out = {}
    for t in rows:
        b = int(case["row_seq"][t])
        pos = int(case["pos"][t])
        if b not in keys_cache:
            keys_cache[b] = seq_keys(case, b)
        kI, kv = keys_cache[b]
        qI, w, q = query_row(case, t)
        sc = indexer_row(qI, w, kI[:pos + 1])
        idx = topk_row(sc.astype(np.float32), case["k"])
        sel = idx[idx >= 0]
        o, lse = sparse_attn_row(q, kv[sel], case["Dv"], case["softmax_scale"])
        out[t] = dict(scores=sc, idx=idx, o=o, lse=lse)
    return out


def attn_rows_on_indices(case: dict, rows, idx_rows, keys_cache=None):
    """Attention of `rows` recomputed on externally given index rows (e.g. a GPU's
    selection): {t: (o [H,Dv], lse [H])}. Index -1 marks padding."""
    keys_cache = {} if keys_cache is None else keys_cache
    res = {}
    for t, idx in zip(rows, idx_rows):
        b = int(case["row_seq"][t])
        if b not in keys_cache:
            keys_cache[b] = seq_keys(case, b)
        _, kv = keys_cache[b]
        _, _, q = query_row(case, t)
        idx = np.asarray(idx)
        sel = idx[idx >= 0]
        res[t] = sparse_attn_row(q, kv[sel], case["Dv"], case["softmax_scale"])
    return res


def indexer_rows(case: dict, rows, keys_cache=None):
    """Indexer scores of `rows` over their causal prefixes: {t: f64[pos+1]}."""
    keys_cache = {} if keys_cache is None else keys_cache
    res = {}
    for t in rows:
        b = int(case["row_seq"][t])
        pos = int(case["pos"][t])
        if b not in keys_cache:
            keys_cache[b] = seq_keys(case, b)
        kI, _ = keys_cache[b]
        qI, w, _ = query_row(case, t)
        res[t] = indexer_row(qI, w, kI[:pos + 1])
    return res


# ---------------------------------------------------------------------------
# cache write: one new token per query row into the paged caches
#   [mundobytes-run] pages of 64 tokens; [mundobytes-kernels] mundobytes.com, the
#   open-kernels paragraph: the indexer kernels come in a paged version;
#   [jdon-indexer] the indexer keys are stored and scored in FP8.
# Readings: one fp32 scale per key token, scale = max|x| / 448 in
# fp32 (1 when the row is all zero); code = the e4m3 value nearest to x / scale
# (fp32 division), ties to the even code, saturating at +-448, the sign kept
# for values that round to zero.

E4M3_MAX = 448.0


def encode_e4m3_rne(y: np.ndarray) -> np.ndarray:
    """e4m3 byte of the representable value nearest to each y (ties to the even
    code), saturating to +-448; NaN -> 0x7F. The non-negative codes 0x00..0x7E
    are the format's finite magnitudes in increasing order, so rounding is a
    search in that table."""
    y = np.asarray(y, dtype=np.float64)
    mags = E4M3_TABLE[:127]                      # codes 0x00 .. 0x7E, increasing
    a = np.minimum(np.abs(y), E4M3_MAX)
    hi = np.clip(np.searchsorted(mags, a, side="left"), 0, 126)   # first magnitude >= a
    lo = np.clip(hi - 1, 0, 126)
    d_lo = a - mags[lo]
    d_hi = mags[hi] - a
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0) & (hi != lo))
    code = np.where(take_hi, hi, lo).astype(np.uint8)
    code = np.where(np.signbit(y), code | 0x80, code).astype(np.uint8)
    return np.where(np.isnan(y), np.uint8(0x7F), code).astype(np.uint8)


def quantize_key_row(x: np.ndarray):
    """(e4m3 bytes, fp32 scale) of one indexer key row, in the kernel's fp32
    arithmetic: scale = float32(max|x|) / float32(448); y = float32(x) / scale."""
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0)
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32) if amax > 0 else np.float32(1.0)
    y = (x32 / scale).astype(np.float32)
    return encode_e4m3_rne(y), np.float32(scale)


def cache_append(case: dict, k_new: np.ndarray, kv_new_bits: np.ndarray, k_pool: np.ndarray,
                 kv_pool_bits: np.ndarray, k_scale: np.ndarray = None):
    """Write row t's new indexer key (quantised) and latent row (bf16 bits, copied)
    at the row's own position pos_t of its sequence. Returns updated copies.

    Paged (page_size 64): k_pool uint8 [pages][8448] = [64 x d_I codes][64 fp32
    scales]; kv_pool_bits uint16 [pages*64][Dk]. Contiguous: k_pool uint8
    [B][n_max][d_I], k_scale float32 [B][n_max], kv_pool_bits [B][n_max][Dk]."""
    k_pool = k_pool.copy()
    kv_pool_bits = kv_pool_bits.copy()
    k_scale = None if k_scale is None else k_scale.copy()
    P = int(case["page_size"])
    d_I = k_new.shape[1]
    for t in range(k_new.shape[0]):
        b = int(case["row_seq"][t])
        pos = int(case["pos"][t])
        codes, sc = quantize_key_row(k_new[t])
        if P:
            page = int(case["page_table"][b][pos // P])
            slot = pos % P
            k_pool[page, slot * d_I:(slot + 1) * d_I] = codes
            k_pool[page, P * d_I + 4 * slot:P * d_I + 4 * slot + 4] = np.frombuffer(
                np.float32(sc).tobytes(), dtype=np.uint8)
            kv_pool_bits[page * P + slot] = kv_new_bits[t]
        else:
            k_pool[b, pos] = codes
            k_scale[b, pos] = sc
            kv_pool_bits[b, pos] = kv_new_bits[t]
    return k_pool, kv_pool_bits, k_scale


# ---------------------------------------------------------------------------
# indexer loss (sparse stage)
#   [jdon-warmup] jdon.com "DeepSeek-V3.2-Exp", warm-up paragraph: the indexer first
#   copies how the main attention distributes its attention, trained with a KL
#   divergence loss; [jdon-sparse-train] same page, sparse-training paragraph: the
#   indexer and the main model are trained together with separated gradients, the
#   indexer optimising only its own scoring loss.
# Readings: the target is the main attention's distribution over the selected set,
# averaged over the heads (each head's softmax sums to 1, so the mean is
# L1-normalised); the indexer's distribution is the softmax of its scores over the
# same set; loss = KL(target || indexer); the indexer's gradient is
# softmax(I) - target, and no gradient reaches the attention inputs.

def indexer_kl_row(q_t: np.ndarray, kv_rows: np.ndarray, scale: float, scores: np.ndarray):
    """(loss, target p, d loss / d scores) for one query row over its selected rows.

    q_t [H, Dk] and kv_rows [m, Dk] as float64 values, scores [m] the indexer
    scores of the same m selected positions."""
    z = scale * (np.asarray(q_t, np.float64) @ np.asarray(kv_rows, np.float64).T)   # [H, m]
    z = z - z.max(axis=1, keepdims=True)
    a = np.exp(z)
    a /= a.sum(axis=1, keepdims=True)            # each head's attention over the selected set
    p = a.mean(axis=0)                           # target: mean over heads, sums to 1
    s = np.asarray(scores, np.float64)
    s = s - s.max()
    q = np.exp(s)
    q /= q.sum()
    nz = p > 0
    loss = float(np.sum(p[nz] * (np.log(p[nz]) - np.log(q[nz]))))
    return loss, p, q - p


# ---------------------------------------------------------------------------
# sparse attention backward (sparse training stage)
#   [jdon-sparse-train] jdon.com "DeepSeek-V3.2-Exp", sparse-training paragraph: the
#   main model is trained on the sparse pattern (k = 2048 entries per query token),
#   separately from the indexer's own loss.
# Readings: the backward of stage 3 with respect to the query heads and the
# selected latent rows, for an upstream gradient dO of the output; the selection
# is piecewise constant and carries no gradient; a position selected by several
# query rows, or twice by one row, receives the sum of its slots' gradients.

def sparse_attn_backward_row(q_t: np.ndarray, kv_rows: np.ndarray, Dv: int, scale: float, dO: np.ndarray):
    """(dq [H, Dk], dkv [m, Dk]): the gradients of sum(dO * o) for one query token,
    o = softmax(scale * q_t . kv_rows^T) @ kv_rows[:, :Dv] per head.

    With P the per-head softmax, dP = dO . v^T and D_h = sum_s P_hs dP_hs:
    dz = P (dP - D), dq = scale dz . kv, and the row gradient is scale dz^T . q
    (key, all Dk dims) plus P^T . dO (value, first Dv dims)."""
    q_t = np.asarray(q_t, np.float64)
    kv_rows = np.asarray(kv_rows, np.float64)
    dO = np.asarray(dO, np.float64)
    z = scale * (q_t @ kv_rows.T)                    # [H, m]
    P = np.exp(z - z.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    v = kv_rows[:, :Dv]
    dP = dO @ v.T                                    # [H, m]
    D = np.sum(P * dP, axis=1, keepdims=True)        # [H, 1] = dO . o per head
    dz = P * (dP - D)
    dq = scale * (dz @ kv_rows)                      # [H, Dk]
    dkv = scale * (dz.T @ q_t)                       # [m, Dk]  through the key
    dkv[:, :Dv] += P.T @ dO                          # through the value
    return dq, dkv


def sparse_attn_backward_seq(q_rows: np.ndarray, kv_seq: np.ndarray, idx: np.ndarray, Dv: int, scale: float,
                             dO: np.ndarray):
    """Backward over the query rows of one sequence: q_rows [R, H, Dk], kv_seq
    [L, Dk] (the sequence's latent rows by position), idx [R, k] (positions, -1 =
    padding), dO [R, H, Dv]. Returns dq [R, H, Dk] and dkv [L, Dk], the latter
    summed over every slot that selected each position. A row with no selected
    position gets dq = 0."""
    R, H, Dk = q_rows.shape
    dq = np.zeros((R, H, Dk))
    dkv = np.zeros((kv_seq.shape[0], Dk))
    for r in range(R):
        sel = np.asarray(idx[r])
        sel = sel[sel >= 0]
        if sel.size == 0:
            continue
        g_q, g_kv = sparse_attn_backward_row(q_rows[r], kv_seq[sel], Dv, scale, dO[r])
        dq[r] = g_q
        np.add.at(dkv, sel, g_kv)
    return dq, dkv
