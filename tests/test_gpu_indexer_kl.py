"""Indexer loss on the selected set (bf16 query rows and latent rows, 128 heads)
against the oracle's KL(p || softmax(I)) per row and its gradient r - p per slot.

Inputs come from the host only: the workload generator's query and latent rows,
selections drawn with a seeded generator (distinct positions in the causal range,
-1 padding anywhere), indexer scores drawn N(0, 2^2), and the attention's per-head
log-sum-exp taken from the oracle. Tolerance: the kernel sums 576 products per
score in fp32 and uses fp32 exponentials, so each p and r carries a relative error
of a few 1e-6; loss within 1e-5 + 1e-3 |loss|, gradient within 2e-6 + 1e-3 |g|."""
import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from sparse_long_context_04_b200 import device as G
from sparse_long_context_04_b200 import dsa as D
from sparse_long_context_04_b200 import workloads as W
from tests.case_utils import case_from_inputs
from tests.gpu_utils import ensure_lib

pytestmark = pytest.mark.gpu


def _selection(case, T, k, seed, holes=False):
    rng = np.random.default_rng(seed)
    idx = np.full((T, k), -1, dtype=np.int32)
    for t in range(T):
        n = int(case["pos"][t]) + 1
        m = min(k, n) if not holes else min(k - k // 4, n)
        sel = np.sort(rng.choice(n, size=m, replace=False)).astype(np.int32)
        if holes:
            slots = np.sort(rng.choice(k, size=m, replace=False))
            idx[t, slots] = sel
        else:
            idx[t, :m] = sel
    return idx


def _run(spec, seed=0, holes=False, rows=None, want_grad=True):
    ensure_lib()
    inp = W.make_inputs(spec)
    case = case_from_inputs(inp)
    dc = G.to_device(inp)
    T, k = inp.T, spec.k
    rows = list(range(T)) if rows is None else list(rows)
    idx = _selection(case, T, k, seed, holes)
    rng = np.random.default_rng(seed + 1)
    scores = rng.normal(0.0, 2.0, size=(T, dc.ld)).astype(np.float32)
    att = O.attn_rows_on_indices(case, range(T), [idx[t] for t in range(T)])
    lse = np.stack([att[t][1] for t in range(T)]).astype(np.float32)
    loss, grad = G.indexer_kl(dc, torch.from_numpy(idx).cuda(), torch.from_numpy(lse).cuda(),
                              torch.from_numpy(scores).cuda(), want_grad=want_grad)
    assert D.dsa_get_device_error() == D.DSA_OK
    loss = loss.cpu().numpy()
    grad = None if grad is None else grad.cpu().numpy()
    cache = {}
    for t in rows:
        b = int(case["row_seq"][t])
        if b not in cache:
            cache[b] = O.seq_keys(case, b)
        _, kv = cache[b]
        _, _, q = O.query_row(case, t)
        live = idx[t] >= 0
        sel = idx[t][live]
        l_ref, _, g_ref = O.indexer_kl_row(q, kv[sel], case["softmax_scale"], scores[t, sel].astype(np.float64))
        assert abs(loss[t] - l_ref) <= 1e-5 + 1e-3 * abs(l_ref), (t, loss[t], l_ref)
        if grad is not None:
            err = np.abs(grad[t][live] - g_ref)
            assert (err <= 2e-6 + 1e-3 * np.abs(g_ref)).all(), (t, float(err.max()))
            assert (grad[t][~live] == 0).all(), t
    return loss


def test_indexer_kl_decode_contiguous_ragged_k():
    # k = 300: nine full 32-slot chunks and a 12-slot tail; one row shorter than k
    _run(W.DECODE_32K.replace(batch=3, lens=(3000, 129, 2053), k=300))


def test_indexer_kl_decode_paged_full_k():
    _run(W.PAGED_DECODE_128K.replace(batch=2, len_range=None, lens=(4100, 2300)), seed=3)


def test_indexer_kl_holes_and_no_gradient():
    _run(W.DECODE_32K.replace(batch=2, lens=(900, 70), k=320), seed=7, holes=True, want_grad=False)


def test_indexer_kl_prefill_rows():
    _run(W.PREFILL_8K.replace(lens=(600,), k=256), seed=11, rows=range(0, 600, 37))


def test_indexer_kl_single_key_rows_have_zero_loss():
    # row 0 selects one position: p = r = 1, so loss and gradient vanish up to rounding
    loss = _run(W.PREFILL_8K.replace(lens=(40,), k=64), seed=2, rows=range(0, 40, 13))
    assert abs(loss[0]) <= 1e-5


def test_indexer_kl_bad_index_is_reported():
    ensure_lib()
    spec = W.DECODE_32K.replace(batch=1, lens=(100,), k=64)
    inp = W.make_inputs(spec)
    dc = G.to_device(inp)
    idx = torch.full((1, 64), -1, dtype=torch.int32, device="cuda")
    idx[0, 0] = 5
    idx[0, 1] = 100          # beyond the query's position 99
    lse = torch.zeros((1, 128), device="cuda")
    scores = torch.zeros((1, dc.ld), device="cuda")
    G.indexer_kl(dc, idx, lse, scores)
    assert D.dsa_get_device_error() == D.DSA_ERR_DEVICE_CHECK
