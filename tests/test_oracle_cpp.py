"""The C++ oracle against the numpy restatement of the same definitions (two
programs written apart: plain loops in double against BLAS matmul and
lexsort), on small cases of every workload shape: contiguous and paged caches,
decode and prefill rows, FP8/bf16 and fp32 inputs. Floating results agree to
rounding (1e-12 relative); selections, codes and cache bytes are identical.
Also: the oracle's results do not depend on its thread count."""
import numpy as np
import pytest

from oracle import dsa_oracle as O
from oracle import numpy_restatement as N
from sparse_long_context_04_b200 import workloads as W
from tests.case_utils import case_from_inputs


def _close(a, b, rel=1e-12):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return a.shape == b.shape and bool(np.all(np.abs(a - b) <= rel * (1.0 + np.abs(b))))


CASES = {
    "tiny_fp32": W.TINY.replace(lens=(96,), k=16),
    "decode_contiguous": W.DECODE_32K.replace(batch=3, lens=(300, 2100, 64), k=256, plant_frac=0.01),
    "decode_paged": W.PAGED_DECODE_128K.replace(batch=3, len_range=None, lens=(700, 130, 2049), k=512),
    "prefill_paged": W.PREFILL_8K.replace(batch=2, lens=(400, 150), q_lens=(100, 150), page_size=64, k=64),
    "prefill_ar1": W.PREFILL_2X32K.replace(lens=(300, 200), k=128),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_forward_rows_agree(name):
    spec = CASES[name]
    case = case_from_inputs(W.make_inputs(spec))
    T = len(case["pos"])
    rows = sorted(set(range(0, T, max(1, T // 12))) | {T - 1})
    got = O.forward_rows(case, rows)
    ref = N.forward_rows(case, rows)
    for t in rows:
        g, r = got[t], ref[t]
        assert _close(g["scores"], r["scores"]), (name, t)
        # the selection on identical float32 scores, and attention on identical indices
        s32 = r["scores"].astype(np.float32)
        assert np.array_equal(O.topk_row(s32, spec.k), N.topk_row(s32, spec.k)), (name, t)
        o, lse = O.attn_rows_on_indices(case, [t], [r["idx"]])[t]
        assert _close(o, r["o"]) and _close(lse, r["lse"]), (name, t)
        assert np.array_equal(O.seq_keys(case, int(case["row_seq"][t]))[1],
                              N.seq_keys(case, int(case["row_seq"][t]))[1]), (name, t)


def test_topk_agrees_on_adversarial_rows():
    rng = np.random.default_rng(3)
    for _ in range(200):
        n = int(rng.integers(1, 300))
        x = rng.choice([0.0, -0.0, 1.0, -1.0, np.inf, -np.inf, np.nan, 0.5], n).astype(np.float32)
        if rng.random() < 0.5:
            x = rng.normal(0, 1, n).astype(np.float32)
        k = int(rng.integers(1, 64))
        assert np.array_equal(O.topk_row(x, k), N.topk_row(x, k))


def test_topk_rows_equals_topk_row():
    rng = np.random.default_rng(4)
    sc = rng.normal(0, 1, (20, 500)).astype(np.float32)
    n = rng.integers(1, 501, 20).astype(np.int32)
    many = O.topk_rows(sc, n, 64)
    for r in range(20):
        assert np.array_equal(many[r], O.topk_row(sc[r, :n[r]], 64))


def test_formats_and_cache_write_agree():
    assert np.array_equal(O.decode_e4m3(np.arange(256, dtype=np.uint8)),
                          N.decode_e4m3(np.arange(256, dtype=np.uint8)), equal_nan=True)
    rng = np.random.default_rng(5)
    y = np.concatenate([rng.normal(0, 100, 5000), [0.0, -0.0, 448.0, 500.0, -1e9, 1e-9, np.nan]])
    assert np.array_equal(O.encode_e4m3_rne(y), N.encode_e4m3_rne(y))
    for _ in range(50):
        x = rng.normal(0, rng.uniform(0.01, 10), 128).astype(np.float32)
        (c1, s1), (c2, s2) = O.quantize_key_row(x), N.quantize_key_row(x)
        assert np.array_equal(c1, c2) and s1 == s2
    spec = CASES["decode_paged"]
    inp = W.make_inputs(spec)
    case = case_from_inputs(inp)
    k_new = rng.normal(0, 1, (3, 128)).astype(np.float32)
    kv_new = rng.integers(0, 2 ** 15, (3, spec.Dk)).astype(np.uint16)
    a = O.cache_append(case, k_new, kv_new, case["k_pages"], case["kv"].reshape(-1, spec.Dk))
    b = N.cache_append(case, k_new, kv_new, case["k_pages"], case["kv"].reshape(-1, spec.Dk))
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_loss_and_backward_agree():
    rng = np.random.default_rng(6)
    H, Dk, Dv, m = 8, 40, 24, 17
    q = rng.normal(0, 1, (H, Dk))
    rows = rng.normal(0, 1, (m, Dk))
    sc = rng.normal(0, 2, m)
    l1, p1, g1 = O.indexer_kl_row(q, rows, 0.3, sc)
    l2, p2, g2 = N.indexer_kl_row(q, rows, 0.3, sc)
    assert _close(l1, l2) and _close(p1, p2) and _close(g1, g2)
    dO = rng.normal(0, 1, (H, Dv))
    a = O.sparse_attn_backward_row(q, rows, Dv, 0.3, dO)
    b = N.sparse_attn_backward_row(q, rows, Dv, 0.3, dO)
    assert _close(a[0], b[0]) and _close(a[1], b[1])
    R, L, k = 5, 30, 7
    qr = rng.normal(0, 1, (R, H, Dk))
    kv = rng.normal(0, 1, (L, Dk))
    idx = rng.integers(-1, L, (R, k)).astype(np.int32)
    idx[2] = -1
    dOr = rng.normal(0, 1, (R, H, Dv))
    a = O.sparse_attn_backward_seq(qr, kv, idx, Dv, 0.3, dOr)
    b = N.sparse_attn_backward_seq(qr, kv, idx, Dv, 0.3, dOr)
    assert _close(a[0], b[0]) and _close(a[1], b[1])


def test_results_do_not_depend_on_thread_count():
    spec = CASES["decode_paged"]
    case = case_from_inputs(W.make_inputs(spec))
    one = O.forward_rows(case, range(3), nthreads=1)
    many = O.forward_rows(case, range(3), nthreads=3)
    for t in range(3):
        for key in ("scores", "idx", "o", "lse"):
            assert np.array_equal(one[t][key], many[t][key]), (t, key)
