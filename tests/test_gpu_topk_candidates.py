"""Top-k from a filtered candidate list (dsa_topk_from_candidates) against the
oracle's top-k over the full row.

The candidates and the 12-bit histograms (of the whole row, or of the candidates
only, as the fused indexer hands them over) are built on the host the way a fused
indexer keeps them: keys arrive tile by tile, each tile is filtered against a
lower bound of the row's threshold bin read from the histogram so far (stale by
a random number of tiles), and the survivors are stored in a shuffled order.
Rows cover ties, signed zeros, infinities, NaN, rows shorter than k, sorted
rows (where the bound never filters), and flat rows whose threshold bin holds
more keys than the kernel stages in shared memory. A histogram that disagrees
with the candidates must be reported as a device check failure."""
import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from sparse_long_context_04_b200 import dsa as D
from tests.gpu_utils import ensure_lib
from tests.test_fused_topk_model import bound_bin, order_key

pytestmark = pytest.mark.gpu


def _candidates(x, k, rng, tile=128):
    """The row's histogram and the positions a streaming filter with a stale bound keeps."""
    bins = (order_key(x) >> 20).astype(np.int64)
    hist = np.zeros(4096, np.int64)
    keep, bound = [], 0
    for t0 in range(0, x.size, tile):
        sl = np.arange(t0, min(x.size, t0 + tile))
        np.add.at(hist, bins[sl], 1)
        keep.append(sl[bins[sl] >= bound])
        if rng.random() < 0.5:
            bound = bound_bin(hist, k)
    keep = np.concatenate(keep)
    rng.shuffle(keep)
    return hist.astype(np.uint32), keep


def _run(rows, k, seed=0, corrupt_row=None, hist_of="all"):
    ensure_lib()
    rng = np.random.default_rng(seed)
    T = len(rows)
    n_max = max(r.size for r in rows)
    cap = n_max
    score = np.zeros((T, cap), np.float32)
    pos = np.full((T, cap), -1, np.int32)
    count = np.zeros(T, np.int32)
    hist = np.zeros((T, 4096), np.uint32)
    for t, x in enumerate(rows):
        h, keep = _candidates(x, k, rng)
        if hist_of == "candidates":   # the fused indexer hands over the candidates' histogram
            h = np.bincount((order_key(x[keep]) >> 20).astype(np.int64), minlength=4096).astype(np.uint32)
        hist[t] = h
        count[t] = keep.size
        score[t, :keep.size] = x[keep]
        pos[t, :keep.size] = keep
    if corrupt_row is not None:
        # five phantom keys in the bin of the row's best key: that bin is at or
        # above the threshold bin, so the candidate counts can no longer agree
        x = rows[corrupt_row]
        top = int(order_key(x).max() >> 20)
        hist[corrupt_row, top] += 5
    seq_lens = torch.tensor([r.size for r in rows], dtype=torch.int32, device="cuda")
    lay = D.Layout(seq_lens, n_max, None)
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    D.dsa_topk_from_candidates(torch.from_numpy(score).cuda(), torch.from_numpy(pos).cuda(),
                               torch.from_numpy(count).cuda(), torch.from_numpy(hist.view(np.int32)).cuda(), k,
                               lay, idx)
    return idx.cpu().numpy()


def _rows(rng, T):
    out = []
    for _ in range(T):
        n = int(rng.choice([1, 100, 2047, 2048, 2049, 20000, 131072]))
        kind = rng.integers(0, 6)
        if kind == 0:
            x = rng.normal(0, 2, n)
        elif kind == 1:
            x = rng.choice([-1.0, 0.0, 0.5, 3.0], n)
        elif kind == 2:
            x = np.sort(rng.normal(0, 1, n))      # rising scores: the bound keeps everything
        elif kind == 3:
            x = rng.choice([0.0, -0.0, np.inf, -np.inf, np.nan, 1.0], n)
        elif kind == 4:
            x = np.full(n, 2.5)                  # one bin (and one key) holds the whole row
        else:
            x = 1.0 + rng.integers(0, 4, n) * 2.0 ** -20   # one bin, four keys: positions decide
        out.append(x.astype(np.float32))
    return out


@pytest.mark.parametrize("hist_of", ["all", "candidates"])
@pytest.mark.parametrize("k", [1, 64, 2048])
def test_topk_from_candidates_equals_full_topk(k, hist_of):
    rng = np.random.default_rng(k)
    rows = _rows(rng, 14)
    got = _run(rows, k, seed=k, hist_of=hist_of)
    assert D.dsa_get_device_error() == D.DSA_OK
    for t, x in enumerate(rows):
        assert np.array_equal(got[t], O.topk_row(x, k)), (t, x.size)


def test_topk_from_candidates_on_indexer_like_rows():
    """Long rows of N(0,1) scores with a few planted high keys, as the decode
    workload's indexer produces them."""
    rng = np.random.default_rng(11)
    rows = []
    for n in (98304, 114688, 131072):
        x = rng.normal(0, 1, n).astype(np.float32)
        x[rng.choice(n, 500, replace=False)] += 4.0
        rows.append(x)
    got = _run(rows, 2048, seed=3)
    assert D.dsa_get_device_error() == D.DSA_OK
    for t, x in enumerate(rows):
        assert np.array_equal(got[t], O.topk_row(x, 2048)), t


def test_inconsistent_histogram_is_reported():
    rng = np.random.default_rng(5)
    rows = [rng.normal(0, 1, 5000).astype(np.float32), rng.normal(0, 1, 3000).astype(np.float32)]
    got = _run(rows, 64, corrupt_row=0)
    assert D.dsa_get_device_error() == D.DSA_ERR_DEVICE_CHECK
    assert np.all(got[0] == -1)
    assert np.array_equal(got[1], O.topk_row(rows[1], 64))   # the other row is unaffected
