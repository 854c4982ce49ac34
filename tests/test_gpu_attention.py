"""bf16 tcgen05 sparse MQA attention (128 heads, 576-wide latent rows, 512-wide
values) against the oracle recomputed on the GPU's own indices: max-abs 2e-2 on
the output and the log-sum-exp. Decode over contiguous and paged caches, split
counts from 1 to 16, prefill with rows shorter than k, index lists with -1 holes,
and dsa_forward."""
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
TOL = 2e-2


def _check_attn(case, idx, out, lse, rows):
    att = O.attn_rows_on_indices(case, rows, [idx[t] for t in rows])
    worst = 0.0
    for t in rows:
        o, l = att[t]
        if (idx[t] >= 0).any():
            e1 = np.abs(out[t].astype(np.float64) - o).max()
            e2 = np.abs(lse[t].astype(np.float64) - l).max()
            assert e1 <= TOL and e2 <= TOL, (t, e1, e2)
            worst = max(worst, e1, e2)
        else:
            assert np.all(out[t] == 0) and np.all(np.isneginf(lse[t])), t
    return worst


def _stages(spec, rows=None):
    ensure_lib()
    inp = W.make_inputs(spec)
    case = case_from_inputs(inp)
    dc = G.to_device(inp)
    scores = G.indexer(dc)
    idx = G.topk(dc, scores)
    out, lse = G.attention(dc, idx)
    assert D.dsa_get_device_error() == D.DSA_OK
    rows = range(inp.T) if rows is None else rows
    _check_attn(case, idx.cpu().numpy(), out.float().cpu().numpy(), lse.cpu().numpy(), rows)
    return inp, case, dc, idx, out, lse


def test_attention_decode_contiguous():
    _stages(W.DECODE_32K.replace(batch=4, lens=(3000, 129, 2053, 64)))


def test_attention_decode_paged():
    _stages(W.PAGED_DECODE_128K.replace(batch=3, len_range=None, lens=(4100, 200, 2048)))


@pytest.mark.parametrize("k", [600, 1300, 4096])
def test_attention_split_counts(k):
    """3, 6 and 16 splits of 256 positions per row (a short last split in the
    first two), merged by the split-merge kernel."""
    _stages(W.PAGED_DECODE_128K.replace(batch=3, len_range=None, lens=(k + 3000, 450, k), k=k))


def test_attention_prefill_short_rows():
    _stages(W.PREFILL_8K.replace(lens=(600,), k=256))


def test_attention_index_holes_and_duplicates():
    ensure_lib()
    spec = W.DECODE_32K.replace(batch=3, lens=(900, 300, 70), k=320)
    inp = W.make_inputs(spec)
    case = case_from_inputs(inp)
    dc = G.to_device(inp)
    rng = np.random.default_rng(5)
    idx = np.full((3, spec.k), -1, dtype=np.int32)
    for b, L in enumerate(spec.lens):
        m = min(L, 250)
        sel = rng.choice(L, size=m, replace=False)
        slots = rng.choice(spec.k, size=m, replace=False)   # -1 anywhere in the list
        idx[b, slots] = sel
    idx[0, 0] = idx[0, 1] = 17                              # a duplicated position counts twice
    idx_d = torch.from_numpy(idx).cuda()
    out, lse = G.attention(dc, idx_d)
    assert D.dsa_get_device_error() == D.DSA_OK
    _check_attn(case, idx, out.float().cpu().numpy(), lse.cpu().numpy(), range(3))


def test_attention_bad_index_is_reported():
    ensure_lib()
    spec = W.DECODE_32K.replace(batch=1, lens=(100,), k=64)
    inp = W.make_inputs(spec)
    dc = G.to_device(inp)
    idx = torch.full((1, 64), -1, dtype=torch.int32, device="cuda")
    idx[0, 0] = 5
    idx[0, 1] = 100          # beyond the query's position 99
    G.attention(dc, idx)
    assert D.dsa_get_device_error() == D.DSA_ERR_DEVICE_CHECK
    assert D.dsa_get_device_error() == D.DSA_OK     # the word is cleared after reading


def test_forward_decode_matches_stages():
    ensure_lib()
    spec = W.PAGED_DECODE_128K.replace(batch=3, len_range=None, lens=(5000, 2048, 300))
    inp = W.make_inputs(spec)
    case = case_from_inputs(inp)
    dc = G.to_device(inp)
    fw = G.Forward(dc)
    out, lse, idx = fw()
    assert D.dsa_get_device_error() == D.DSA_OK
    scores = G.indexer(dc)
    idx2 = G.topk(dc, scores)
    out2, lse2 = G.attention(dc, idx2)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx2)
    assert torch.equal(out, out2) and torch.equal(lse, lse2)
    ref = O.forward_rows(case, range(3))
    for t in range(3):   # end to end against the oracle's own selection
        assert np.array_equal(idx[t].cpu().numpy(), ref[t]["idx"]), t
        assert np.abs(out[t].float().cpu().numpy() - ref[t]["o"]).max() <= TOL


def test_forward_prefill_end_to_end():
    ensure_lib()
    spec = W.PREFILL_2X32K.replace(lens=(700, 300), k=256)
    inp = W.make_inputs(spec)
    case = case_from_inputs(inp)
    dc = G.to_device(inp)
    out, lse, idx = G.Forward(dc)()
    assert D.dsa_get_device_error() == D.DSA_OK
    scores = G.indexer(dc).cpu().numpy()
    ix = idx.cpu().numpy()
    for t in range(inp.T):
        pos = int(case["pos"][t])
        assert np.array_equal(ix[t], O.topk_row(scores[t, :pos + 1], spec.k)), t
    _check_attn(case, ix, out.float().cpu().numpy(), lse.cpu().numpy(), range(0, inp.T, 5))
