"""Exactness of the fused indexer -> top-k selection, checked on numpy models
(no GPU, no kernel).

The producer-and-finisher model: keys arrive tile by tile from several CTAs in an
arbitrary interleaving; each tile is filtered against a lower bound on the row's
k-th largest key that may be stale by any number of tiles (the floor of the
highest 12-bit radix bin with at least k keys at or above it in the row's
histogram so far); the survivors are appended in arrival order; a final step
takes the threshold bin from the complete histogram, ranks that bin's candidates
by (key descending, position ascending) and emits the positions in ascending
order. The finishing kernel's own steps are then emulated digit by digit (two
10-bit key digits and two 9-bit position digits inside the threshold bin). Both
must equal the oracle's top-k for every row, including ties, -0 against +0,
infinities, NaN, rows shorter than k and score orders that defeat the filter
(scores rising with position)."""
import numpy as np
import pytest

from oracle import dsa_oracle as O

BITS = 12


def order_key(x):
    """Larger float -> larger key; -0 and +0 share a key; NaN below -inf."""
    u = np.asarray(x, np.float32).view(np.uint32).copy()
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    u[u == 0x80000000] = 0
    key = np.where(u & 0x80000000, ~u, u | 0x80000000).astype(np.uint32)
    key[nan] = 0
    return key


def bound_bin(hist, k):
    """Highest bin b with at least k keys in bins >= b (0 while fewer than k)."""
    suffix = np.cumsum(hist[::-1])[::-1]
    ok = np.nonzero(suffix >= k)[0]
    return int(ok.max()) if ok.size else 0


def fused_select(scores, k, P, rng, tile=128):
    n = scores.size
    key = order_key(scores)
    bins = (key >> (32 - BITS)).astype(np.int64)
    nt = -(-n // tile)
    per = -(-nt // P)
    queues = [list(range(c * per, min(nt, (c + 1) * per))) for c in range(P)]
    hist = np.zeros(1 << BITS, np.int64)
    published = 0                     # the row's bound word
    seen_by = [0] * P                 # the bound each CTA last read
    cand = []
    while any(queues):
        c = rng.choice([i for i in range(P) if queues[i]])
        t = queues[c].pop(0)
        if rng.random() < 0.5:        # re-read the bound now, or filter with a stale one
            seen_by[c] = published
        pos = np.arange(t * tile, min(n, (t + 1) * tile))
        np.add.at(hist, bins[pos], 1)
        cand.extend(pos[bins[pos] >= seen_by[c]].tolist())
        if rng.random() < 0.3:        # some CTA refreshes the published bound
            published = max(published, bound_bin(hist, k))
    m = min(k, n)
    cand = np.array(cand, np.int64)
    B = bound_bin(hist, m)
    above = cand[bins[cand] > B]
    at = cand[bins[cand] == B]
    order = np.lexsort((at, -key[at].astype(np.int64)))   # key descending, position ascending
    chosen = np.sort(np.concatenate([above, at[order[:m - above.size]]]))
    out = np.full(k, -1, np.int32)
    out[:m] = chosen
    return out, cand.size


def _rows(rng):
    n = int(rng.choice([1, 5, 127, 128, 129, 1000, 4000]))
    kind = rng.integers(0, 6)
    if kind == 0:
        x = rng.normal(0, 2, n)
    elif kind == 1:
        x = rng.choice([-1.0, 0.0, 0.5, 3.0], n)                      # heavy ties
    elif kind == 2:
        x = np.sort(rng.normal(0, 1, n))                               # rising: every key passes the filter
    elif kind == 3:
        x = rng.choice([0.0, -0.0, np.inf, -np.inf, np.nan, 1.0], n)  # signed zeros, infinities, NaN
    elif kind == 4:
        x = np.full(n, 2.5)                                            # all equal
    else:
        x = np.abs(rng.normal(0, 1, n)) * rng.choice([1e-30, 1.0, 1e30], n)  # wide range
    return x.astype(np.float32)


@pytest.mark.parametrize("seed", range(12))
def test_streaming_selection_equals_the_oracle(seed):
    rng = np.random.default_rng(seed)
    for _ in range(25):
        x = _rows(rng)
        k = int(rng.choice([1, 7, 64, 300, 2048]))
        P = int(rng.choice([1, 3, 9]))
        got, _ = fused_select(x, k, P, rng)
        assert np.array_equal(got, O.topk_row(x, k)), (seed, x.size, k, P)


def test_candidates_are_few_on_unordered_scores():
    # i.i.d. scores: the survivors stay near k (1 + ln(n / k)), far below n
    rng = np.random.default_rng(99)
    x = rng.normal(0, 1, 60_000).astype(np.float32)
    got, ncand = fused_select(x, 2048, 9, rng)
    assert np.array_equal(got, O.topk_row(x, 2048))
    assert ncand < 0.25 * x.size, ncand


# ---------------------------------------------------------------------------
# The finishing kernel's own steps (topk_candidates_kernel): the threshold bin
# from the histogram, two 10-bit key digits and two 9-bit position digits inside
# it, and the bitmap of selected positions, emulated digit by digit.

def _find_digit(cnt, need, from_top):
    before = 0
    for d in (range(1023, -1, -1) if from_top else range(1024)):
        if before < need <= before + cnt[d]:
            return d, before
        before += cnt[d]
    raise AssertionError("no digit")


def kernel_steps(x, hist, cand, k):
    n = x.size
    m = min(k, n)
    above, B, above_b = 0, None, None
    for b in range(4095, -1, -1):
        if above < m <= above + hist[b]:
            B, above_b = b, above
        above += hist[b]
    keys = order_key(x)
    chosen = np.zeros(n, bool)
    ties = []
    for s in cand:
        key = int(keys[s])
        if key >> 20 > B:
            chosen[s] = True
        elif key >> 20 == B:
            ties.append((key, int(s)))
    assert chosen.sum() == above_b and len(ties) == hist[B]
    need_ties = m - above_b
    kstar, pstar = 0, (1 << 18) - 1
    if need_ties < len(ties):
        prefix, need = B << 20, need_ties
        for shift, pmask in ((10, 0xFFF00000), (0, 0xFFFFFC00)):
            cnt = np.zeros(1024, np.int64)
            for key, _ in ties:
                if key & pmask == prefix:
                    cnt[(key >> shift) & 1023] += 1
            d, rem = _find_digit(cnt, need, True)
            prefix |= d << shift
            need -= rem
        kstar = prefix
        for p in range(2):
            shift = 9 if p == 0 else 0
            cnt = np.zeros(1024, np.int64)
            for key, s in ties:
                if key == kstar and (p == 0 or s >> 9 == pstar >> 9):
                    cnt[(s >> shift) & 511] += 1
            d, rem = _find_digit(cnt, need, False)
            pstar = (d << 9) | 511 if p == 0 else (pstar & ~511) | d
            need -= rem
    for key, s in ties:
        if need_ties >= len(ties) or key > kstar or (key == kstar and s <= pstar):
            chosen[s] = True
    out = np.full(k, -1, np.int32)
    sel = np.nonzero(chosen)[0]
    assert sel.size == m
    out[:m] = sel
    return out


@pytest.mark.parametrize("seed", range(4))
def test_finishing_kernel_steps_equal_the_oracle(seed):
    rng = np.random.default_rng(100 + seed)
    for _ in range(30):
        x = _rows(rng)
        k = int(rng.choice([1, 7, 64, 2048]))
        bins = (order_key(x) >> 20).astype(np.int64)
        hist = np.bincount(bins, minlength=4096)
        bound = bound_bin(hist, k) if rng.random() < 0.5 else 0
        cand = np.nonzero(bins >= bound)[0]
        rng.shuffle(cand)
        assert np.array_equal(kernel_steps(x, hist, cand, k), O.topk_row(x, k)), (x.size, k)
