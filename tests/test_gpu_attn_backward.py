"""Sparse-attention backward (bf16, 128 heads, 576-wide latent rows, 512-wide
values) against the oracle's gradients of sum(dO * o) with respect to the query
heads and the selected latent rows.

Inputs come from the host only: the workload generator's query and latent rows,
selections drawn with a seeded generator (distinct positions in the causal range
unless a test plants a duplicate, -1 padding anywhere), dO drawn N(0, 1) and
rounded to bf16, and the forward output (rounded to bf16) and log-sum-exp from the
oracle. Tolerance: the kernel feeds P and dz to the tensor cores as bf16 (relative
rounding 2^-9) and takes D = dO . o from the bf16 output, so each gradient carries
an error of a few 2^-9 of the call's typical gradient size, whatever the row's own
size (a row with one selected key has an exact dq of 0 but a rounding residue).
Per row (dq) and per sequence (dkv) the max-abs error must stay within 1.5e-2 of
the larger of that row's (sequence's) max-abs reference and the median of those
maxima over the call. Rows and positions that nothing selected must stay exactly
zero."""
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
REL = 1.5e-2


def _selection(case, T, k, seed, holes=False, dup=False):
    rng = np.random.default_rng(seed)
    idx = np.full((T, k), -1, dtype=np.int32)
    for t in range(T):
        n = int(case["pos"][t]) + 1
        m = min(k - k // 4 if holes else k, n)
        sel = np.sort(rng.choice(n, size=m, replace=False)).astype(np.int32)
        slots = np.sort(rng.choice(k, size=m, replace=False)) if holes else np.arange(m)
        idx[t, slots] = sel
        if dup and m >= 2:
            idx[t, slots[1]] = idx[t, slots[0]]      # one position counted twice
    return idx


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16)


def _phys_row(inp, b, s):
    ps = inp.spec.page_size
    if ps:
        return int(inp.page_table[b, s // ps]) * ps + s % ps
    return b * inp.n_max + s


def _run(spec, seed=0, holes=False, dup=False):
    ensure_lib()
    inp = W.make_inputs(spec)
    case = case_from_inputs(inp)
    dc = G.to_device(inp)
    T, k, H, Dk, Dv = inp.T, spec.k, spec.H, spec.Dk, spec.Dv
    idx = _selection(case, T, k, seed, holes, dup)
    rng = np.random.default_rng(seed + 1)
    dO = _bf16(rng.normal(size=(T, H, Dv)))
    att = O.attn_rows_on_indices(case, range(T), [idx[t] for t in range(T)])
    out = _bf16(np.stack([att[t][0] for t in range(T)]))
    lse = torch.from_numpy(np.stack([att[t][1] for t in range(T)]).astype(np.float32))
    dq = torch.zeros((T, H, Dk), dtype=torch.float32, device="cuda")
    dkv = torch.zeros(tuple(dc.kv.shape), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(D.dsa_sparse_mqa_attn_backward_workspace_size(T), 256), dtype=torch.uint8, device="cuda")
    D.dsa_sparse_mqa_attn_backward(dc.q, dc.kv, torch.from_numpy(idx).cuda(), dc.layout, out.cuda(), dO.cuda(),
                                   lse.cuda(), dq, dkv, spec.softmax_scale, ws)
    assert D.dsa_get_device_error() == D.DSA_OK
    dq = dq.cpu().numpy()
    dkv = dkv.view(-1, Dk).cpu().numpy()
    dO64 = dO.float().numpy().astype(np.float64)
    touched = np.zeros(dkv.shape[0], dtype=bool)
    rows_of = {}
    for t in range(T):
        rows_of.setdefault(int(case["row_seq"][t]), []).append(t)
    ref = {}
    for b, rows in rows_of.items():
        _, kv = O.seq_keys(case, b)
        q_rows = np.stack([O.query_row(case, t)[2] for t in rows])
        ref[b] = O.sparse_attn_backward_seq(q_rows, kv, idx[rows], Dv, case["softmax_scale"], dO64[rows])
    q_scale = np.median([np.abs(g).max() for b in ref for g in ref[b][0]])
    kv_scale = np.median([np.abs(ref[b][1]).max() for b in ref])
    for b, rows in rows_of.items():
        g_q, g_kv = ref[b]
        for r, t in enumerate(rows):
            if (idx[t] >= 0).any():
                err = np.abs(dq[t] - g_q[r]).max()
                assert err <= REL * max(np.abs(g_q[r]).max(), q_scale), (t, err, np.abs(g_q[r]).max(), q_scale)
            else:
                assert np.all(dq[t] == 0), t
        L = int(case["seq_lens"][b])
        phys = np.array([_phys_row(inp, b, s) for s in range(L)])
        got = dkv[phys]
        err = np.abs(got - g_kv).max()
        assert err <= REL * max(np.abs(g_kv).max(), kv_scale), (b, err, np.abs(g_kv).max())
        sel = np.unique(np.concatenate([idx[t][idx[t] >= 0] for t in rows]))
        assert np.all(got[np.setdiff1d(np.arange(L), sel)] == 0), b
        touched[phys] = True
    assert np.all(dkv[~touched] == 0)       # rows of no sequence in this call


def test_attn_backward_decode_contiguous_ragged_k():
    # k = 300: two full 128-slot CTAs and a 44-slot tail; one row shorter than k
    _run(W.DECODE_32K.replace(batch=3, lens=(3000, 129, 2053), k=300))


def test_attn_backward_decode_paged_full_k():
    _run(W.PAGED_DECODE_128K.replace(batch=2, len_range=None, lens=(4100, 2300)), seed=3)


def test_attn_backward_holes_and_a_duplicate():
    _run(W.DECODE_32K.replace(batch=2, lens=(900, 70), k=320), seed=7, holes=True, dup=True)


def test_attn_backward_prefill_rows_share_positions():
    # 300 rows of one sequence select overlapping positions: dkv sums across rows
    _run(W.PREFILL_8K.replace(lens=(300,), k=128), seed=11)


def test_attn_backward_bad_index_is_reported():
    ensure_lib()
    spec = W.DECODE_32K.replace(batch=1, lens=(100,), k=64)
    inp = W.make_inputs(spec)
    dc = G.to_device(inp)
    idx = torch.full((1, 64), -1, dtype=torch.int32, device="cuda")
    idx[0, 0] = 5
    idx[0, 1] = 100          # beyond the query's position 99
    z = torch.zeros((1, 128, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 128), device="cuda")
    dq = torch.zeros((1, 128, 576), device="cuda")
    dkv = torch.zeros(tuple(dc.kv.shape), dtype=torch.float32, device="cuda")
    ws = torch.empty(D.dsa_sparse_mqa_attn_backward_workspace_size(1), dtype=torch.uint8, device="cuda")
    D.dsa_sparse_mqa_attn_backward(dc.q, dc.kv, idx, dc.layout, z, z, lse, dq, dkv, spec.softmax_scale, ws)
    assert D.dsa_get_device_error() == D.DSA_ERR_DEVICE_CHECK
