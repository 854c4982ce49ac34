"""The fused indexer -> top-k on decode rows: dsa_indexer_candidates (the indexer
writing each row's order-key histograms and a filtered candidate list instead of
its scores), dsa_topk_from_candidates, and dsa_forward, which chains them for
decode rows when asked to (topk_path = DSA_TOPK_FUSED).

Checked against the GPU's own unfused scores (dsa_indexer_scores, the same
indexer arithmetic):
  - every candidate's score equals the unfused score at its position, bit for
    bit; positions are distinct and causal; every key at or above the row's
    threshold bin is a candidate; each row's 12-bit histogram counts exactly its
    candidates;
  - dsa_forward's selection equals the oracle's top-k of the unfused scores on
    every row, and its attention output equals the attention on that selection;
  - on rows built to defeat the filter: equal scores everywhere (one bin holds
    the whole row, every key is a candidate), scores that rise with position
    (each new key beats the ones before it) and scores that fall."""
import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from sparse_long_context_04_b200 import device as G
from sparse_long_context_04_b200 import dsa as D
from sparse_long_context_04_b200 import workloads as W
from tests.gpu_utils import ensure_lib
from tests.test_fused_topk_model import order_key

pytestmark = pytest.mark.gpu


def _producer(dc, k):
    T, cap = dc.T, dc.ld
    dev = dc.q.device
    hist = torch.full((T, 4096), 7, dtype=torch.int32, device=dev)     # not zero: the call clears it
    cs = torch.empty((T, cap), dtype=torch.float32, device=dev)
    cp = torch.empty((T, cap), dtype=torch.int32, device=dev)
    cnt = torch.full((T,), 7, dtype=torch.int32, device=dev)
    D.dsa_indexer_candidates(dc.q_idx, dc.q_scale, dc.k_idx, dc.k_scale, dc.w, dc.layout, k, hist, cs, cp, cnt)
    torch.cuda.synchronize()
    assert D.dsa_get_device_error_site() == (D.DSA_OK, 0)
    return hist.cpu().numpy(), cs.cpu().numpy(), cp.cpu().numpy(), cnt.cpu().numpy()


def _check(dc, k):
    pos = dc.inp.pos.numpy()
    scores = G.indexer(dc).cpu().numpy()
    hist, cs, cp, cnt = _producer(dc, k)
    kept = 0
    for t in range(dc.T):
        n = int(pos[t]) + 1
        row = scores[t, :n]
        bins = (order_key(row) >> 20).astype(np.int64)
        c = int(cnt[t])
        assert 0 < c <= dc.ld, (t, c)
        p = cp[t, :c]
        assert np.unique(p).size == c and p.min() >= 0 and p.max() < n, t
        assert np.array_equal(cs[t, :c].view(np.uint32), row[p].view(np.uint32)), t
        assert np.array_equal(hist[t], np.bincount(bins[p], minlength=4096)), t   # the candidates' histogram
        sel = O.topk_row(row, k)
        sel = sel[sel >= 0]
        thr_bin = int((order_key(row[sel]) >> 20).min())
        must = np.nonzero(bins >= thr_bin)[0]
        assert np.isin(must, p).all(), t
        kept += c
    return scores, kept


def _forward_check(dc, scores):
    s = dc.inp.spec
    pos = dc.inp.pos.numpy()
    out, lse, idx = G.Forward(dc, topk_path=D.DSA_TOPK_FUSED)()
    torch.cuda.synchronize()
    assert D.dsa_get_device_error_site() == (D.DSA_OK, 0)
    ix = idx.cpu().numpy()
    for t in range(dc.T):
        assert np.array_equal(ix[t], O.topk_row(scores[t, :int(pos[t]) + 1], s.k)), t
    ref_out, ref_lse = G.attention(dc, idx)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16)) and torch.equal(lse, ref_lse)


@pytest.mark.parametrize("k", [64, 300, 2048])
def test_fused_paged_decode(k):
    ensure_lib()
    spec = W.PAGED_DECODE_128K.replace(batch=5, len_range=None, lens=(6000, 2048, 300, 40000, 2049), k=k)
    dc = G.to_device(W.make_inputs(spec))
    scores, kept = _check(dc, k)
    _forward_check(dc, scores)


def test_fused_contiguous_decode():
    ensure_lib()
    spec = W.DECODE_32K.replace(batch=4, lens=(5000, 64, 2047, 9000))
    dc = G.to_device(W.make_inputs(spec))
    scores, _ = _check(dc, spec.k)
    _forward_check(dc, scores)


def _adversarial(kind):
    """A contiguous decode case whose rows' keys share one code row; the per-token
    scales then order the scores: all equal, rising or falling with position."""
    spec = W.DECODE_32K.replace(batch=3, lens=(20000, 3000, 70000))
    inp = W.make_inputs(spec)
    B, n_max = inp.k_idx.shape[0], inp.n_max
    for b in range(B):
        # the key code row the query scores highest, so that the scores are not all zero
        inp.k_idx[b, :] = inp.q_idx[b, int(torch.argmax(inp.w[b]))][None, :]
        L = int(inp.seq_lens[b])
        ramp = torch.linspace(0.5, 2.0, L)
        inp.k_scale[b, :L] = {"equal": torch.ones(L), "rising": ramp, "falling": ramp.flip(0)}[kind]
    return G.to_device(inp)


@pytest.mark.parametrize("kind", ["equal", "rising", "falling"])
def test_fused_adversarial_score_orders(kind):
    ensure_lib()
    dc = _adversarial(kind)
    scores, kept = _check(dc, dc.inp.spec.k)
    if kind == "equal":
        assert kept == int((dc.inp.pos + 1).sum())   # one bin: nothing can be filtered out
    _forward_check(dc, scores)
