"""Pins of the CPU oracle against things other than itself: published format
tables, hand-worked cases, closed forms, library routines on special cases,
brute-force enumeration and invariants the method's definition implies."""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _floats(tokens):
    return [float(x) for x in tokens]


# ----------------------------------------------------------------- formats

def test_e4m3_against_ocp_table():
    for line in open(os.path.join(GOLD, "e4m3_ocp_table.txt")):
        if line.startswith("#") or not line.strip():
            continue
        b, v = line.split()
        got = O.e4m3_value(int(b, 16))
        want = float(v)
        if math.isnan(want):
            assert math.isnan(got)
        else:
            assert got == want and math.copysign(1, got) == math.copysign(1, want), (b, got, want)


def test_e4m3_table_against_torch_cast():
    # torch's float8_e4m3fn -> float32 conversion is an independent implementation
    allb = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = allb.view(torch.float8_e4m3fn).to(torch.float32).numpy().astype(np.float64)
    mine = O.decode_e4m3(np.arange(256, dtype=np.uint8))
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(mine))
    assert np.array_equal(ref[~nan], mine[~nan])
    assert nan.sum() == 2  # 0x7F and 0xFF only


def test_bf16_decode_against_torch():
    g = torch.Generator().manual_seed(3)
    x = (torch.randn(4096, generator=g) * 100).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.decode_bf16(bits), x.to(torch.float64).numpy())


def test_fp8_per_token_roundtrip_bound():
    from sparse_long_context_04_b200.workloads import encode_e4m3_per_token
    rng = np.random.default_rng(0)
    x = rng.standard_normal((64, 128)).astype(np.float32)
    q8, s = encode_e4m3_per_token(x)
    xd = O.dequant(q8.numpy(), s.numpy())
    # RNE to 3 mantissa bits: relative error <= 2^-4 for normals, absolute
    # error <= 2^-10 * s in the subnormal range
    err = np.abs(xd - x)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * s.numpy()[:, None]) * (1 + 1e-6)
    assert np.all(err <= bound)
    # the per-token maximum maps to 448 exactly
    assert np.allclose(np.abs(xd).max(axis=1), np.abs(x).max(axis=1), rtol=1e-6)


# ----------------------------------------------------------------- indexer

def _hand_indexer():
    d = {}
    for line in open(os.path.join(GOLD, "indexer_hand_example.txt")):
        if line.startswith("#") or not line.strip():
            continue
        key, *vals = line.split()
        d[key] = np.array(_floats(vals))
    return d


def test_indexer_hand_example_and_reading_guards():
    d = _hand_indexer()
    q = d["q"].reshape(2, 2)
    k = d["k"].reshape(3, 2)
    I = O.indexer_row(q, d["w"], k)
    assert np.array_equal(I, d["I"])
    assert not np.array_equal(I, d["relu_after_sum"])
    assert not np.array_equal(I, d["no_relu"])


def test_indexer_single_head_nonnegative_is_plain_matmul():
    rng = np.random.default_rng(1)
    q = np.abs(rng.standard_normal((1, 32)))
    keys = np.abs(rng.standard_normal((50, 32)))
    I = O.indexer_row(q, np.ones(1), keys)
    ref = torch.from_numpy(keys) @ torch.from_numpy(q[0])   # library matmul
    assert np.allclose(I, ref.numpy(), rtol=1e-13, atol=0)


def test_indexer_relu_identities():
    """relu(x) - relu(-x) = x and relu(x) + relu(-x) = |x| per head: negating one
    head's query moves the score by w_j * (q_j . k); summing the score of q and -q
    gives sum_j w_j |q_j . k|. A ReLU placed anywhere else breaks both."""
    rng = np.random.default_rng(2)
    H, d, n = 5, 16, 40
    q = rng.standard_normal((H, d))
    w = rng.standard_normal(H)
    keys = rng.standard_normal((n, d))
    base = O.indexer_row(q, w, keys)
    for j in range(H):
        qn = q.copy()
        qn[j] = -qn[j]
        diff = base - O.indexer_row(qn, w, keys)
        assert np.allclose(diff, w[j] * np.einsum("sd,d->s", keys, q[j]), atol=1e-12)
    both = base + O.indexer_row(-q, w, keys)
    ref = np.abs(np.einsum("sd,hd->sh", keys, q)) @ w
    assert np.allclose(both, ref, atol=1e-12)


def test_indexer_linear_in_w_and_positively_homogeneous():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((4, 8))
    keys = rng.standard_normal((30, 8))
    w1, w2 = rng.standard_normal(4), rng.standard_normal(4)
    assert np.allclose(O.indexer_row(q, w1 + w2, keys),
                       O.indexer_row(q, w1, keys) + O.indexer_row(q, w2, keys), atol=1e-12)
    assert np.allclose(O.indexer_row(2.5 * q, w1, keys), 2.5 * O.indexer_row(q, w1, keys), atol=1e-12)
    assert np.allclose(O.indexer_row(q, w1, 0.25 * keys), 0.25 * O.indexer_row(q, w1, keys), atol=1e-12)


def test_indexer_scale_folding():
    """Per-token FP8 scales multiply the dequantised vectors: scores from (bytes,
    scales) equal scores from pre-scaled vectors with unit scales."""
    rng = np.random.default_rng(5)
    qb = rng.integers(0, 256, size=(3, 4, 16)).astype(np.uint8)
    kb = rng.integers(0, 256, size=(20, 16)).astype(np.uint8)
    qb[(qb & 0x7F) == 0x7F] = 0  # no NaN bytes
    kb[(kb & 0x7F) == 0x7F] = 0
    sq = rng.uniform(0.01, 2, size=3).astype(np.float32)
    sk = rng.uniform(0.01, 2, size=20).astype(np.float32)
    w = rng.standard_normal(4)
    keys = O.dequant(kb, sk)
    for t in range(3):
        q = O.dequant(qb[t][None], sq[t:t + 1])[0]
        a = O.indexer_row(q, w, keys)
        b = sq[t] * (np.maximum(O.decode_e4m3(kb) @ O.decode_e4m3(qb[t]).T * sk[:, None], 0) @ w)
        assert np.allclose(a, b, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------- top-k

def _brute_topk(v, k):
    """Enumerate every subset of size m = min(k, n); keep the unique one whose
    members all precede all non-members under (score desc, index asc)."""
    n = len(v)
    m = min(k, n)

    def before(a, b):  # does index a precede index b?
        va, vb = v[a], v[b]
        na, nb = math.isnan(va), math.isnan(vb)
        if na != nb:
            return nb          # a number precedes NaN
        if not na and va != vb:
            return va > vb
        return a < b

    winners = []
    for sub in itertools.combinations(range(n), m):
        rest = set(range(n)) - set(sub)
        if all(before(a, b) for a in sub for b in rest):
            winners.append(sub)
    assert len(winners) == 1
    out = list(winners[0]) + [-1] * (k - m)
    return np.array(out, dtype=np.int32)


def test_topk_hand_examples():
    for line in open(os.path.join(GOLD, "topk_hand_examples.txt")):
        if line.startswith("#") or not line.strip():
            continue
        k, sc, exp = [p.strip() for p in line.split("|")]
        v = np.array([float(x) for x in sc.split()], dtype=np.float32)
        want = np.array([int(x) for x in exp.split()], dtype=np.int32)
        assert np.array_equal(O.topk_row(v, int(k)), want), line


def test_topk_brute_force_small_rows():
    rng = np.random.default_rng(7)
    pool = np.array([0.0, -0.0, 1.0, 1.0, -1.0, 2.5, np.inf, -np.inf, np.nan, 3.0, 1e-30],
                    dtype=np.float32)
    for trial in range(400):
        n = int(rng.integers(1, 11))
        if trial % 2:
            v = rng.choice(pool, size=n)
        else:
            v = rng.integers(-2, 3, size=n).astype(np.float32)
        k = int(rng.integers(1, 13))
        assert np.array_equal(O.topk_row(v, k), _brute_topk([float(x) for x in v], k)), (v, k)


def test_topk_short_rows_select_everything():
    rng = np.random.default_rng(8)
    for n in (1, 5, 63, 64):
        v = rng.standard_normal(n).astype(np.float32)
        out = O.topk_row(v, 64)
        assert np.array_equal(out[:n], np.arange(n)) and np.all(out[n:] == -1)


def test_topk_threshold_tie_across_k():
    v = np.zeros(100, dtype=np.float32)
    v[[3, 50, 97]] = 1.0
    out = O.topk_row(v, 10)
    assert np.array_equal(out, np.array([0, 1, 2, 3, 4, 5, 6, 7, 50, 97], dtype=np.int32))


# ----------------------------------------------------------------- attention

def test_attention_hand_example():
    d = {}
    for line in open(os.path.join(GOLD, "attention_hand_example.txt")):
        if line.startswith("#") or not line.strip():
            continue
        key, *vals = line.split()
        d[key] = np.array(_floats(vals))
    o, lse = O.sparse_attn_row(d["q"].reshape(1, 2), d["rows"].reshape(2, 2), 1, 1.0)
    assert abs(o[0, 0] - d["o"][0]) < 1e-15 and abs(lse[0] - d["lse"][0]) < 1e-15


def test_attention_against_torch_sdpa():
    """Selected-row attention equals a library softmax-attention on the gathered
    rows with key = whole row, value = first Dv dims."""
    rng = np.random.default_rng(9)
    H, Dk, Dv, m = 6, 24, 10, 37
    q = rng.standard_normal((H, Dk))
    rows = rng.standard_normal((m, Dk))
    scale = 0.3
    o, lse = O.sparse_attn_row(q, rows, Dv, scale)
    qt = torch.from_numpy(q)[:, None, :]
    kt = torch.from_numpy(rows)[None].expand(H, m, Dk)
    vt = torch.from_numpy(rows[:, :Dv])[None].expand(H, m, Dv)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)[:, 0]
    assert np.allclose(o, ref.numpy(), atol=1e-12)
    ref_lse = torch.logsumexp(scale * (torch.from_numpy(q) @ torch.from_numpy(rows).T), dim=1)
    assert np.allclose(lse, ref_lse.numpy(), atol=1e-12)


def test_attention_single_row_and_two_row_closed_forms():
    rng = np.random.default_rng(10)
    q = rng.standard_normal((3, 8))
    r = rng.standard_normal((2, 8))
    o1, l1 = O.sparse_attn_row(q, r[:1], 5, 0.7)
    assert np.array_equal(o1, np.broadcast_to(r[0, :5], (3, 5)))
    assert np.allclose(l1, 0.7 * q @ r[0], atol=1e-14)
    o2, l2 = O.sparse_attn_row(q, r, 5, 0.7)
    z = 0.7 * q @ r.T
    a = 1.0 / (1.0 + np.exp(z[:, 1] - z[:, 0]))
    assert np.allclose(o2, a[:, None] * r[0, :5] + (1 - a)[:, None] * r[1, :5], atol=1e-14)
    assert np.allclose(l2, np.log(np.exp(z[:, 0]) + np.exp(z[:, 1])), atol=1e-14)


def test_attention_permutation_invariant():
    rng = np.random.default_rng(11)
    q = rng.standard_normal((4, 16))
    rows = rng.standard_normal((20, 16))
    o, l = O.sparse_attn_row(q, rows, 8, 0.25)
    p = rng.permutation(20)
    o2, l2 = O.sparse_attn_row(q, rows[p], 8, 0.25)
    assert np.allclose(o, o2, atol=1e-12) and np.allclose(l, l2, atol=1e-12)


def dense_causal_mqa_online(q_t, kv_prefix, Dv, scale):
    """Dense causal MQA for one token as a one-key-at-a-time online softmax: a
    different algorithm from the oracle's two-pass softmax over a selection,
    written here so that the invariant below checks the oracle against something
    other than itself."""
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


def test_dsa_with_k_at_least_L_is_dense_causal_mqa():
    from sparse_long_context_04_b200.workloads import TINY, make_inputs
    from tests.case_utils import case_from_inputs
    spec = TINY.replace(lens=(40,), k=64)
    case = case_from_inputs(make_inputs(spec))
    res = O.forward_rows(case, range(40))
    kI, kv = O.seq_keys(case, 0)
    for t in (0, 1, 17, 39):
        assert np.array_equal(res[t]["idx"][:t + 1], np.arange(t + 1))
        _, _, q = O.query_row(case, t)
        o, l = dense_causal_mqa_online(q, kv[:t + 1], spec.Dv, spec.softmax_scale)
        assert np.allclose(res[t]["o"], o, atol=1e-12) and np.allclose(res[t]["lse"], l, atol=1e-12)


# ----------------------------------------------------------------- causality, paging

def test_causality_future_data_does_not_change_row():
    from sparse_long_context_04_b200.workloads import TINY, make_inputs
    from tests.case_utils import case_from_inputs
    spec = TINY.replace(lens=(96,), k=16)
    case = case_from_inputs(make_inputs(spec))
    rows = [10, 50, 95]
    a = O.forward_rows(case, rows)
    rng = np.random.default_rng(12)
    for t in rows[:2]:
        case2 = dict(case)
        case2["k_idx"] = case["k_idx"].copy()
        case2["kv"] = case["kv"].copy()
        case2["k_idx"][0, t + 1:] = rng.standard_normal(case2["k_idx"][0, t + 1:].shape)
        case2["kv"][0, t + 1:] = rng.standard_normal(case2["kv"][0, t + 1:].shape)
        b = O.forward_rows(case2, [t])[t]
        for key in ("scores", "idx", "o", "lse"):
            assert np.array_equal(a[t][key], b[key])


def test_paged_and_contiguous_layouts_agree():
    from sparse_long_context_04_b200.workloads import PAGED_DECODE_128K, make_inputs
    from tests.case_utils import case_from_inputs
    spec = PAGED_DECODE_128K.replace(batch=3, len_range=None, lens=(200, 64, 129), k=128,
                                     plant_frac=0.05)
    paged = case_from_inputs(make_inputs(spec))
    contig = case_from_inputs(make_inputs(spec.replace(page_size=0)))
    for b in range(3):
        kp, vp = O.seq_keys(paged, b)
        kc, vc = O.seq_keys(contig, b)
        assert np.array_equal(kp, kc) and np.array_equal(vp, vc)
    ra = O.forward_rows(paged, range(3))
    rb = O.forward_rows(contig, range(3))
    for t in range(3):
        for key in ("scores", "idx", "o", "lse"):
            assert np.array_equal(ra[t][key], rb[t][key])


def test_paged_addressing_against_hand_built_pool():
    """Build a tiny paged pool by hand (page size 4, a chosen page order) and
    check the oracle's logical view recovers the rows in position order."""
    P, d = 4, 16
    L = 10
    rng = np.random.default_rng(13)
    kb = rng.integers(0, 0x70, size=(L, d)).astype(np.uint8)
    sc = rng.uniform(0.5, 2, size=L).astype(np.float32)
    kv = rng.integers(0, 2 ** 14, size=(L, 6)).astype(np.uint16)
    order = [2, 0, 1]       # logical page i lives in physical page order[i]
    pages = np.zeros((3, P * d + 4 * P), dtype=np.uint8)
    kvpool = np.zeros((3, P, 6), dtype=np.uint16)
    for s in range(L):
        pg, sl = order[s // P], s % P
        pages[pg, sl * d:(sl + 1) * d] = kb[s]
        pages[pg, P * d + 4 * sl:P * d + 4 * sl + 4] = np.frombuffer(sc[s].tobytes(), np.uint8)
        kvpool[pg, sl] = kv[s]
    case = dict(fp8=True, page_size=P, d_I=d, seq_lens=np.array([L]), page_table=np.array([order]),
                k_pages=pages, kv=kvpool)
    kI, kvr = O.seq_keys(case, 0)
    assert np.array_equal(kI, O.decode_e4m3(kb) * sc[:, None].astype(np.float64))
    assert np.array_equal(kvr, O.decode_bf16(kv))


# ---------------------------------------------------------------------------
# cache write: e4m3 encoding and per-token quantisation (pinned to the format's
# grid, not to the oracle's own search)

def _brute_e4m3(y: float) -> int:
    """Nearest finite e4m3 code by exhaustive search over the 254 finite codes of
    y's sign (saturating), ties to the code with an even mantissa."""
    a = min(abs(y), 448.0)
    best, best_d = None, None
    for c in range(0x7F):                      # non-negative finite codes
        v = O.e4m3_value(c)
        d = abs(v - a)
        if best is None or d < best_d or (d == best_d and c % 2 == 0):
            best, best_d = c, d
    return best | (0x80 if np.signbit(y) else 0)


def test_e4m3_encode_round_trips_every_finite_code():
    for c in list(range(0x7F)) + list(range(0x80, 0xFF)):
        assert int(O.encode_e4m3_rne(np.array([O.e4m3_value(c)]))[0]) == c, hex(c)


def test_e4m3_encode_midpoints_go_to_the_even_code():
    for c in range(0x7E):
        lo, hi = O.e4m3_value(c), O.e4m3_value(c + 1)
        mid = (lo + hi) / 2
        even = c if c % 2 == 0 else c + 1
        assert int(O.encode_e4m3_rne(np.array([mid]))[0]) == even, (hex(c), mid)
        assert int(O.encode_e4m3_rne(np.array([-mid]))[0]) == even | 0x80
        # a hair off the midpoint picks the nearer neighbour
        eps = (hi - lo) * 1e-3
        assert int(O.encode_e4m3_rne(np.array([mid - eps]))[0]) == c
        assert int(O.encode_e4m3_rne(np.array([mid + eps]))[0]) == c + 1


def test_e4m3_encode_matches_exhaustive_search():
    rng = np.random.default_rng(7)
    ys = np.concatenate([rng.standard_normal(400) * 60, rng.standard_normal(200) * 0.01,
                         [0.0, -0.0, 448.0, 449.0, 464.0, 1e6, -1e6, 2.0 ** -9, 2.0 ** -10, -2.0 ** -10]])
    got = O.encode_e4m3_rne(ys)
    want = np.array([_brute_e4m3(float(v)) for v in ys], dtype=np.uint8)
    assert np.array_equal(got, want)
    assert int(O.encode_e4m3_rne(np.array([np.nan]))[0]) == 0x7F


def test_quantize_key_row_scale_and_error_bound():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(128).astype(np.float32) * 3
    codes, sc = O.quantize_key_row(x)
    assert sc == np.float32(np.max(np.abs(x)) / np.float32(448.0))
    i = int(np.argmax(np.abs(x)))
    assert codes[i] in (0x7E, 0xFE)                       # the largest element maps to +-448
    back = O.decode_e4m3(codes) * np.float64(sc)
    big = np.abs(x) >= 2.0 ** -6 * sc                      # normal range: 3 mantissa bits
    assert np.all(np.abs(back[big] - x[big]) <= np.abs(x[big]) / 16 + 1e-12)
    z_codes, z_sc = O.quantize_key_row(np.zeros(128, np.float32))
    assert z_sc == 1.0 and not z_codes.any()


def test_cache_append_writes_only_the_rows_own_slot():
    rng = np.random.default_rng(5)
    P, d_I, Dk, pages = 64, 128, 576, 6
    case = {"page_size": P, "row_seq": np.array([0, 1]), "pos": np.array([70, 5]),
            "page_table": np.array([[4, 1], [3, 0]])}
    k_pool = rng.integers(0, 256, (pages, P * d_I + 4 * P), dtype=np.uint8)
    kv_pool = rng.integers(0, 65536, (pages * P, Dk), dtype=np.uint16)
    k_new = rng.standard_normal((2, d_I)).astype(np.float32)
    kv_new = rng.integers(0, 65536, (2, Dk), dtype=np.uint16)
    k2, kv2, _ = O.cache_append(case, k_new, kv_new, k_pool, kv_pool)
    # row 0: position 70 -> page_table[0][1] = 1, slot 6; row 1: position 5 -> page 3, slot 5
    c0, s0 = O.quantize_key_row(k_new[0])
    c1, s1 = O.quantize_key_row(k_new[1])
    assert np.array_equal(k2[1, 6 * d_I:7 * d_I], c0)
    assert np.array_equal(k2[3, 5 * d_I:6 * d_I], c1)
    assert k2[1, P * d_I + 24:P * d_I + 28].view(np.float32)[0] == s0
    assert k2[3, P * d_I + 20:P * d_I + 24].view(np.float32)[0] == s1
    assert np.array_equal(kv2[1 * P + 6], kv_new[0]) and np.array_equal(kv2[3 * P + 5], kv_new[1])
    changed = np.argwhere(k2 != k_pool)
    assert set(map(tuple, changed[:, :1].tolist())) <= {(1,), (3,)}
    assert (kv2 != kv_pool).any(axis=1).sum() <= 2


# ---------------------------------------------------------------------------
# indexer loss: pinned by the properties KL must have and by finite differences

def _kl_case(seed, H=4, Dk=16, m=9):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((H, Dk)), rng.standard_normal((m, Dk)), rng.standard_normal(m) * 2


def test_indexer_kl_target_is_a_distribution_and_loss_is_nonnegative():
    q, kv, s = _kl_case(1)
    loss, p, g = O.indexer_kl_row(q, kv, 0.3, s)
    assert np.isclose(p.sum(), 1.0) and (p > 0).all()
    assert loss >= 0.0
    assert np.isclose(g.sum(), 0.0)              # both distributions sum to 1


def test_indexer_kl_vanishes_when_scores_are_log_target_plus_a_constant():
    q, kv, _ = _kl_case(2)
    _, p, _ = O.indexer_kl_row(q, kv, 0.3, np.zeros(kv.shape[0]))
    loss, _, g = O.indexer_kl_row(q, kv, 0.3, np.log(p) + 7.5)
    assert abs(loss) < 1e-12 and np.abs(g).max() < 1e-12


def test_indexer_kl_single_head_two_keys_closed_form():
    # one head, two keys: p = softmax(z), q = softmax(s); KL written out by hand
    q = np.array([[1.0, 0.0]])
    kv = np.array([[2.0, 0.0], [0.0, 0.0]])
    scale = 0.5
    z = np.array([1.0, 0.0])
    p = np.exp(z) / np.exp(z).sum()
    s = np.array([0.2, -0.4])
    qq = np.exp(s) / np.exp(s).sum()
    want = p[0] * np.log(p[0] / qq[0]) + p[1] * np.log(p[1] / qq[1])
    loss, pp, g = O.indexer_kl_row(q, kv, scale, s)
    assert np.isclose(loss, want) and np.allclose(pp, p) and np.allclose(g, qq - p)


def test_indexer_kl_gradient_matches_finite_differences():
    q, kv, s = _kl_case(3)
    _, _, g = O.indexer_kl_row(q, kv, 0.3, s)
    eps = 1e-6
    for i in range(len(s)):
        d = np.zeros_like(s)
        d[i] = eps
        num = (O.indexer_kl_row(q, kv, 0.3, s + d)[0] - O.indexer_kl_row(q, kv, 0.3, s - d)[0]) / (2 * eps)
        assert abs(num - g[i]) < 1e-7, (i, num, g[i])


def test_indexer_kl_target_is_the_mean_of_the_heads_attention():
    # heads that attend to disjoint keys: the target splits the mass evenly between them
    q = np.array([[50.0, 0.0], [0.0, 50.0]])
    kv = np.array([[1.0, 0.0], [0.0, 1.0]])
    _, p, _ = O.indexer_kl_row(q, kv, 1.0, np.zeros(2))
    assert np.allclose(p, [0.5, 0.5], atol=1e-12)
    # one sharp head, one flat head: the mean of the softmaxes (0.75, 0.25), not the
    # softmax of the summed logits (1, 0) nor one head's attention
    q = np.array([[50.0, 0.0], [0.0, 0.0]])
    _, p, _ = O.indexer_kl_row(q, kv, 1.0, np.zeros(2))
    assert np.allclose(p, [0.75, 0.25], atol=1e-12)


# ---------------------------------------------------------------------------
# sparse attention backward: pinned by finite differences of the forward, an
# independent autograd implementation, a one-key closed form and a translation
# invariance of the key-only dimensions.

def _attn_loss(q, kv, Dv, scale, dO):
    o, _ = O.sparse_attn_row(q, kv, Dv, scale)
    return float(np.sum(dO * o))


def test_attn_backward_matches_central_differences():
    rng = np.random.default_rng(41)
    H, m, Dk, Dv, scale = 3, 4, 7, 5, 0.37
    q = rng.normal(size=(H, Dk))
    kv = rng.normal(size=(m, Dk))
    dO = rng.normal(size=(H, Dv))
    dq, dkv = O.sparse_attn_backward_row(q, kv, Dv, scale, dO)
    eps = 1e-6
    for arr, grad in ((q, dq), (kv, dkv)):
        num = np.zeros_like(arr)
        for ix in np.ndindex(arr.shape):
            a0 = arr[ix]
            arr[ix] = a0 + eps
            lp = _attn_loss(q, kv, Dv, scale, dO)
            arr[ix] = a0 - eps
            lm = _attn_loss(q, kv, Dv, scale, dO)
            arr[ix] = a0
            num[ix] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8)


def test_attn_backward_matches_torch_autograd_fp64():
    rng = np.random.default_rng(42)
    H, m, Dk, Dv, scale = 8, 20, 40, 32, 1 / np.sqrt(40)
    q = rng.normal(size=(H, Dk))
    kv = rng.normal(size=(m, Dk))
    dO = rng.normal(size=(H, Dv))
    tq = torch.tensor(q, dtype=torch.float64, requires_grad=True)
    tkv = torch.tensor(kv, dtype=torch.float64, requires_grad=True)
    o = torch.softmax(scale * tq @ tkv.T, dim=1) @ tkv[:, :Dv]
    (o * torch.tensor(dO, dtype=torch.float64)).sum().backward()
    dq, dkv = O.sparse_attn_backward_row(q, kv, Dv, scale, dO)
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dkv, tkv.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_attn_backward_one_key_closed_form():
    # one selected row: P = 1 and o = v for every head, so nothing reaches the
    # query or the key; the value receives the heads' summed output gradient
    rng = np.random.default_rng(43)
    H, Dk, Dv = 4, 9, 6
    q, kv, dO = rng.normal(size=(H, Dk)), rng.normal(size=(1, Dk)), rng.normal(size=(H, Dv))
    dq, dkv = O.sparse_attn_backward_row(q, kv, Dv, 0.5, dO)
    np.testing.assert_allclose(dq, 0.0, atol=1e-14)
    np.testing.assert_allclose(dkv[0, :Dv], dO.sum(axis=0), rtol=1e-13)
    np.testing.assert_allclose(dkv[0, Dv:], 0.0, atol=1e-14)


def test_attn_backward_key_only_dims_sum_to_zero():
    # adding one vector c to the key-only dims (Dv..Dk) of every selected row shifts
    # each head's scores by a constant and leaves o unchanged: the rows' gradients in
    # those dims sum to zero
    rng = np.random.default_rng(44)
    H, m, Dk, Dv = 5, 11, 12, 8
    q, kv, dO = rng.normal(size=(H, Dk)), rng.normal(size=(m, Dk)), rng.normal(size=(H, Dv))
    _, dkv = O.sparse_attn_backward_row(q, kv, Dv, 0.3, dO)
    np.testing.assert_allclose(dkv[:, Dv:].sum(axis=0), 0.0, atol=1e-12)
    assert np.abs(dkv[:, Dv:]).max() > 1e-3      # not zero row by row


def test_attn_backward_seq_accumulates_duplicates_and_skips_padding():
    # finite differences through the whole sequence: rows that share positions, a
    # position selected twice by one row, -1 padding and a row with nothing selected
    rng = np.random.default_rng(45)
    R, H, L, Dk, Dv, scale = 3, 2, 6, 5, 3, 0.45
    q = rng.normal(size=(R, H, Dk))
    kv = rng.normal(size=(L, Dk))
    dO = rng.normal(size=(R, H, Dv))
    idx = np.array([[0, 2, 2, -1], [-1, 1, 2, 5], [-1, -1, -1, -1]])

    def loss():
        tot = 0.0
        for r in range(R):
            sel = idx[r][idx[r] >= 0]
            if sel.size:
                tot += _attn_loss(q[r], kv[sel], Dv, scale, dO[r])
        return tot

    dq, dkv = O.sparse_attn_backward_seq(q, kv, idx, Dv, scale, dO)
    eps = 1e-6
    for arr, grad in ((q, dq), (kv, dkv)):
        num = np.zeros_like(arr)
        for ix in np.ndindex(arr.shape):
            a0 = arr[ix]
            arr[ix] = a0 + eps
            lp = loss()
            arr[ix] = a0 - eps
            lm = loss()
            arr[ix] = a0
            num[ix] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8)
    assert np.all(dq[2] == 0) and np.all(dkv[[3, 4]] == 0)
