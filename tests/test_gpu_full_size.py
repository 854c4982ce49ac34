"""Parity at the workloads' full sizes, through dsa_forward (the same kernels the
benchmark times), on sampled query rows the oracle computes one by one:
  - indexer: the row's every causal score within rel 1e-2 / abs 1e-3,
  - top-k: bit-exact against the oracle's selection on the GPU's own scores,
    and equal to the selection dsa_forward made,
  - attention: output and log-sum-exp within 2e-2, recomputed on the GPU's indices.
Sampled rows include the short-row boundary (pos = k-1, k) and sequence edges.
On the prefill workloads the selection is also checked on every row: the GPU's
scores of each chunk of 4096 rows (a prefill call of its own over the same cache)
against the oracle's top-k of those scores, bit for bit."""
import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from sparse_long_context_04_b200 import device as G
from sparse_long_context_04_b200 import dsa as D
from sparse_long_context_04_b200 import workloads as W
from tests.case_utils import case_from_inputs
from tests.gpu_utils import ensure_lib, indexer_close

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
TOL = 2e-2


def _rows(spec, inp):
    T = inp.T
    if spec.mode == "decode":
        return list(range(T))
    rng = np.random.default_rng(spec.seed)
    pos = inp.pos.numpy()
    must = {0, T - 1}
    for t in range(T):
        if pos[t] in (spec.k - 1, spec.k, spec.k + 1) or t == 0 or (t > 0 and pos[t] == 0):
            must.add(t)
            if t > 0:
                must.add(t - 1)
    extra = set(int(x) for x in rng.choice(T, size=8, replace=False))
    return sorted(must | extra)


def _run(name):
    ensure_lib()
    spec = W.WORKLOADS[name]
    inp = W.make_inputs(spec)
    case = case_from_inputs(inp)
    dc = G.to_device(inp)
    fw = G.Forward(dc)
    out, lse, idx = fw()
    torch.cuda.synchronize()
    assert D.dsa_get_device_error_site() == (D.DSA_OK, 0)
    rows = _rows(spec, inp)
    rows_t = torch.tensor(rows, dtype=torch.long, device=dc.q.device)
    scores = G.indexer(dc)                       # standalone call: same kernel, all rows
    sc = scores.index_select(0, rows_t).cpu().numpy()
    del scores
    ix = idx.index_select(0, rows_t).cpu().numpy()
    o_np = out.index_select(0, rows_t).float().cpu().numpy()
    l_np = lse.index_select(0, rows_t).cpu().numpy()
    assert D.dsa_get_device_error() == D.DSA_OK
    cache = {}
    ref = O.indexer_rows(case, rows, cache)
    att = O.attn_rows_on_indices(case, rows, list(ix), cache)
    for r, t in enumerate(rows):
        pos = int(case["pos"][t])
        got = sc[r, :pos + 1]
        ok, err, nbad = indexer_close(got, ref[t])
        assert ok, (name, t, err, nbad)
        assert np.array_equal(ix[r], O.topk_row(got, spec.k)), (name, t)
        o, l = att[t]
        e1 = np.abs(o_np[r] - o).max()
        e2 = np.abs(l_np[r] - l).max()
        assert e1 <= TOL and e2 <= TOL, (name, t, e1, e2)
    if spec.mode == "prefill":
        assert _topk_every_row(dc, idx) == inp.T
    return len(rows)


def _topk_every_row(dc, idx, chunk=4096):
    """Every prefill row's selection against the oracle's top-k of the GPU's scores.
    Rows r0..r1-1 of sequence b (positions p0..p1-1) are scored as a prefill call of
    their own: one sequence of length p1 whose last r1-r0 tokens are the queries."""
    inp, spec = dc.inp, dc.inp.spec
    dev = dc.q.device
    cu = inp.cu_q.tolist()
    pos = inp.pos.numpy()
    checked = 0
    for b in range(len(cu) - 1):
        for r0 in range(cu[b], cu[b + 1], chunk):
            r1 = min(cu[b + 1], r0 + chunk)
            lay = D.Layout(torch.tensor([int(pos[r1 - 1]) + 1], dtype=torch.int32, device=dev), dc.layout.c.n_max,
                           torch.tensor([0, r1 - r0], dtype=torch.int32, device=dev))
            scores = torch.empty((r1 - r0, dc.ld), dtype=torch.float32, device=dev)
            D.dsa_indexer_scores(dc.q_idx[r0:r1], dc.q_scale[r0:r1], dc.k_idx[b:b + 1], dc.k_scale[b:b + 1],
                                 dc.w[r0:r1], lay, scores)
            torch.cuda.synchronize()
            assert D.dsa_get_device_error() == D.DSA_OK
            want = O.topk_rows(scores.cpu().numpy(), (pos[r0:r1] + 1).astype(np.int32), spec.k)
            got = idx[r0:r1].cpu().numpy()
            bad = np.nonzero((got != want).any(axis=1))[0]
            assert bad.size == 0, (spec.name, int(r0 + bad[0]))
            checked += r1 - r0
            del scores
    return checked


def test_full_decode_b32_ctx32k():
    assert _run("decode_b32_ctx32k") == 32


def test_full_prefill_L8192():
    assert _run("prefill_L8192") >= 10


def test_full_prefill_2x32768_ar1():
    assert _run("prefill_2x32768_ar1") >= 10


def test_full_paged_decode_b16_ctx96k_128k():
    assert _run("paged_decode_b16_ctx96k_128k") == 16
