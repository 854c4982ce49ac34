"""Top-k selection on the GPU is bit-exact against the oracle's selection on
the same fp32 score rows: random, tie-heavy, signed-zero, NaN and -inf rows, for
single-CTA and cluster (2..8 CTAs per row) launches, decode and prefill rows."""
import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from sparse_long_context_04_b200 import dsa as D
from tests.gpu_utils import ensure_lib

pytestmark = pytest.mark.gpu


def _rows(rng, B, n):
    kinds = []
    out = np.empty((B, n), dtype=np.float32)
    for b in range(B):
        kind = b % 6
        if kind == 0:
            r = rng.standard_normal(n)
        elif kind == 1:
            r = rng.integers(-3, 4, size=n).astype(np.float64)       # heavy ties
        elif kind == 2:
            r = np.where(rng.random(n) < 0.5, 0.0, -0.0) * 1.0
            r[rng.random(n) < 0.01] = 1.0                            # few above a zero plateau
        elif kind == 3:
            r = np.full(n, 2.5)                                      # all equal
        elif kind == 4:
            r = rng.standard_normal(n)
            r[rng.random(n) < 0.05] = np.nan
            r[rng.random(n) < 0.05] = -np.inf
            r[rng.random(n) < 0.01] = np.inf
        else:
            r = np.abs(rng.standard_normal(n)) * 1e-3 + 7.0           # same exponent, mantissa-only differences
        out[b] = r.astype(np.float32)
        if kind == 2:
            out[b][np.signbit(r)] = -0.0
    return out


@pytest.mark.parametrize("lens,k", [
    ((100, 37, 64), 128),                    # every row shorter than k
    ((5000, 2049, 4096, 3000, 2048, 9000), 2048),
    ((32768,) * 4, 2048),
    ((131072, 98304, 120000, 111111), 2048),  # cluster of 8 per row
    ((70000, 1), 64),
])
def test_topk_decode_rows_bit_exact(lens, k):
    ensure_lib()
    rng = np.random.default_rng(sum(lens) + k)
    B = len(lens)
    n_max = max(lens)
    ld = (n_max + 3) // 4 * 4 + 4
    host = _rows(rng, B, ld)
    scores = torch.from_numpy(host).cuda()
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    lay = D.Layout(seq, n_max)
    idx = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    D.dsa_topk(scores, k, lay, idx)
    assert D.dsa_get_device_error() == D.DSA_OK
    got = idx.cpu().numpy()
    for b, L in enumerate(lens):
        want = O.topk_row(host[b, :L], k)
        assert np.array_equal(got[b], want), (b, L, np.nonzero(got[b] != want)[0][:10])


def test_topk_prefill_rows_bit_exact():
    ensure_lib()
    rng = np.random.default_rng(11)
    lens = (3000, 700)
    q_lens = (3000, 300)          # second sequence: only its last 300 tokens are queries
    k = 1024
    T = sum(q_lens)
    ld = 3000
    host = _rows(rng, T, ld)
    scores = torch.from_numpy(host).cuda()
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    cu_q = torch.tensor([0, 3000, 3300], dtype=torch.int32, device="cuda")
    lay = D.Layout(seq, max(lens), cu_q)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    D.dsa_topk(scores, k, lay, idx)
    assert D.dsa_get_device_error() == D.DSA_OK
    got = idx.cpu().numpy()
    for t in list(range(0, 3000, 7)) + list(range(3000, 3300)):
        pos = t if t < 3000 else 400 + (t - 3000)
        want = O.topk_row(host[t, :pos + 1], k)
        assert np.array_equal(got[t], want), t


def test_topk_zero_rows_is_a_no_op():
    ensure_lib()
    seq = torch.tensor([5], dtype=torch.int32, device="cuda")
    cu_q = torch.tensor([0, 0], dtype=torch.int32, device="cuda")
    lay = D.Layout(seq, 5, cu_q)
    scores = torch.zeros((1, 8), device="cuda")
    idx = torch.full((1, 4), 3, dtype=torch.int32, device="cuda")
    D.dsa_topk(scores, 4, lay, idx, T=0)
    torch.cuda.synchronize()
    assert idx.cpu().tolist() == [[3, 3, 3, 3]]


@pytest.mark.parametrize("lens", [(131072, 100000, 65536, 40000), (20000, 6000, 2500)])
def test_topk_few_ties_at_the_threshold_bit_exact(lens):
    """Scores rounded to 1e-3: a handful of keys tie at the k-th best value, so the
    selection must take the lowest positions among them (ties resolved on the
    candidate list, not by the full-radix fallback)."""
    ensure_lib()
    k = 2048
    rng = np.random.default_rng(sum(lens))
    B = len(lens)
    n_max = max(lens)
    ld = (n_max + 3) // 4 * 4
    host = np.round(rng.standard_normal((B, ld)), 3).astype(np.float32)
    scores = torch.from_numpy(host).cuda()
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    lay = D.Layout(seq, n_max)
    idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
    D.dsa_topk(scores, k, lay, idx)
    assert D.dsa_get_device_error() == D.DSA_OK
    got = idx.cpu().numpy()
    partial_ties = 0
    for b, L in enumerate(lens):
        row = host[b, :L]
        want = O.topk_row(row, k)
        assert np.array_equal(got[b], want), (b, L)
        kth = np.sort(row)[::-1][k - 1]
        partial_ties += (row == kth).sum() > k - (row > kth).sum()
    assert partial_ties >= 2  # the case under test: only some of the tied keys are taken


@pytest.mark.parametrize("lens", [(131072, 120000, 40000, 9000)])
def test_topk_sorted_rows_bit_exact(lens):
    """Rising and falling rows: the best keys crowd into one end of the row, so a
    few warps hold all the keys at or above the threshold bin (more than their
    key lists take) while the others hold none."""
    ensure_lib()
    k = 2048
    rng = np.random.default_rng(sum(lens))
    B = len(lens)
    n_max = max(lens)
    ld = (n_max + 3) // 4 * 4
    host = np.sort(rng.standard_normal((B, ld)), axis=1).astype(np.float32)
    host[1::2] = host[1::2, ::-1]
    scores = torch.from_numpy(np.ascontiguousarray(host)).cuda()
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    lay = D.Layout(seq, n_max)
    idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
    D.dsa_topk(scores, k, lay, idx)
    assert D.dsa_get_device_error() == D.DSA_OK
    got = idx.cpu().numpy()
    for b, L in enumerate(lens):
        assert np.array_equal(got[b], O.topk_row(host[b, :L], k)), b
