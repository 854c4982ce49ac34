"""Prefill over paged caches through dsa_forward, the layout every rank of the
multi-GPU prefill runs.

1. A two-sequence paged prefill with fewer query rows than keys in one sequence
   (its rows are the last tokens): indexer within rel 1e-2 / abs 1e-3 on every
   row, top-k bit-exact against the oracle's top-k of the GPU's own scores on
   every row, attention within 2e-2 on sampled rows recomputed on the GPU's
   indices.
2. One long sequence split for two ranks (zig-zag chunks, the pools gathered
   without a collective): each rank's two-piece paged prefill on this GPU must
   give the same selection, output and log-sum-exp, bit for bit, as the
   unsharded contiguous prefill, since every row sees the same keys in the same
   tiles."""
import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from sparse_long_context_04_b200 import device as G
from sparse_long_context_04_b200 import dsa as D
from sparse_long_context_04_b200 import prefill_shard as S
from sparse_long_context_04_b200 import workloads as W
from tests.case_utils import case_from_inputs
from tests.gpu_utils import ensure_lib, indexer_close

pytestmark = pytest.mark.gpu
TOL = 2e-2


def test_forward_paged_prefill_matches_oracle():
    ensure_lib()
    spec = W.PREFILL_8K.replace(batch=2, lens=(3000, 1500), q_lens=(700, 1500), page_size=64)
    inp = W.make_inputs(spec)
    case = case_from_inputs(inp)
    dc = G.to_device(inp)
    out, lse, idx = G.Forward(dc)()
    scores = G.indexer(dc)
    torch.cuda.synchronize()
    assert D.dsa_get_device_error_site() == (D.DSA_OK, 0)
    sc = scores.cpu().numpy()
    ix = idx.cpu().numpy()
    rows = list(range(inp.T))
    ref = O.indexer_rows(case, rows)
    for t in rows:
        pos = int(case["pos"][t])
        got = sc[t, :pos + 1]
        ok, err, nbad = indexer_close(got, ref[t])
        assert ok, (t, err, nbad)
        assert np.array_equal(ix[t], O.topk_row(got, spec.k)), t
    rng = np.random.default_rng(1)
    sample = sorted({0, 699, 700, 701, inp.T - 1} | set(int(x) for x in rng.choice(inp.T, 24, replace=False)))
    att = O.attn_rows_on_indices(case, sample, [ix[t] for t in sample])
    o_np = out.float().cpu().numpy()
    l_np = lse.cpu().numpy()
    for t in sample:
        o, l = att[t]
        assert np.abs(o_np[t] - o).max() <= TOL and np.abs(l_np[t] - l).max() <= TOL, t


def _pool(pl, inp):
    L = int(inp.seq_lens[0])
    cache = (inp.k_idx[0, :L], inp.k_scale[0, :L], inp.kv[0, :L])
    parts = [S.pack_local_pages(pl, r, *cache) for r in range(pl.world)]
    return torch.cat([p[0] for p in parts]), torch.cat([p[1] for p in parts])


def test_sharded_rank_layouts_equal_the_unsharded_prefill():
    ensure_lib()
    L, world = 5000, 2
    spec = W.PREFILL_8K.replace(lens=(L,))
    inp = W.make_inputs(spec)
    dc = G.to_device(inp)
    full_out, full_lse, full_idx = G.Forward(dc)()
    pl = S.plan(L, world)
    k_pool, kv_pool = _pool(pl, inp)
    k_pool, kv_pool = k_pool.cuda(), kv_pool.cuda()
    for rank in range(world):
        pos = torch.from_numpy(pl.positions(rank))
        lens, cu, pt = pl.layout_arrays(rank)
        seq_lens, cu_q, page_table = (torch.from_numpy(a).cuda() for a in (lens, cu, pt))
        lay = D.Layout(seq_lens, L, cu_q, page_table, S.PAGE, pl.pool_pages)
        T = int(pos.numel())
        q_idx, q_scale, w, q = (x[pos].contiguous().cuda() for x in (inp.q_idx, inp.q_scale, inp.w, inp.q))
        out = torch.empty((T, spec.H, spec.Dv), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((T, spec.H), dtype=torch.float32, device="cuda")
        idx = torch.empty((T, spec.k), dtype=torch.int32, device="cuda")
        args = D.forward_args(q_idx, q_scale, k_pool, None, w, q, kv_pool, spec.k, spec.softmax_scale, lay, out,
                              lse, idx)
        ws = torch.empty(D.dsa_forward_workspace_size(args), dtype=torch.uint8, device="cuda")
        D.dsa_forward(args, ws)
        torch.cuda.synchronize()
        assert D.dsa_get_device_error_site() == (D.DSA_OK, 0), rank
        rows = pos.cuda()
        assert torch.equal(idx, full_idx.index_select(0, rows)), rank
        assert torch.equal(out.view(torch.int16), full_out.index_select(0, rows).view(torch.int16)), rank
        assert torch.equal(lse, full_lse.index_select(0, rows)), rank
