"""Multi-GPU prefill sharding, host side on CPU: the zig-zag split covers every
position once with equal causal cost per rank, the page table maps the
sequence's logical pages into the gathered pool, two and three gloo ranks
all-gather their pages into byte-identical pools that hold every token's cache
rows, and the oracle run on one rank's two-piece paged layout gives exactly the
unsharded results for the same positions."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import dsa_oracle as O
from sparse_long_context_04_b200 import prefill_shard as S
from sparse_long_context_04_b200 import workloads as W
from tests.case_utils import case_from_inputs, to_np


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("L", [64, 1000, 4096, 6000])
def test_split_covers_every_position_once(L, world):
    pl = S.plan(L, world)
    assert pl.C % S.PAGE == 0 and pl.n_chunks * pl.C >= L
    pos = np.concatenate([pl.positions(r) for r in range(world)])
    assert np.array_equal(np.sort(pos), np.arange(L))
    pt = pl.page_table()
    assert len(set(pt.tolist())) == pl.max_pages and pt.min() >= 0 and pt.max() < pl.pool_pages


@pytest.mark.parametrize("world", [1, 2, 4, 8])
def test_split_balances_causal_cost(world):
    # when the chunks tile the sequence exactly every rank visits the same number of keys
    L = 2 * world * 256
    costs = [S.plan(L, world).cost(r) for r in range(world)]
    assert len(set(costs)) == 1 and sum(costs) == L * (L + 1) // 2
    # ragged lengths stay close: the last chunk is short
    for L in (1000, 6000, 100_000):
        costs = [S.plan(L, world).cost(r) for r in range(world)]
        assert max(costs) <= 1.15 * (sum(costs) / world), (L, costs)


def test_page_table_example():
    # L = 1000, two ranks: C = 256 (4 pages); rank 0 holds chunks 0 and 3, rank 1 chunks 1 and 2
    pl = S.plan(1000, 2)
    assert pl.C == 256 and pl.chunks(0) == (0, 3) and pl.chunks(1) == (1, 2)
    assert pl.page_table().tolist() == [0, 1, 2, 3, 8, 9, 10, 11, 12, 13, 14, 15, 4, 5, 6, 7]
    lens, cu, pt = pl.layout_arrays(0)
    assert lens.tolist() == [256, 1000] and cu.tolist() == [0, 256, 256 + 232]
    assert pt.shape == (2, 16)


def _spec(L):
    return W.PREFILL_8K.replace(lens=(L,), k=64)


def _cache(inp):
    L = int(inp.seq_lens[0])
    return inp.k_idx[0, :L], inp.k_scale[0, :L], inp.kv[0, :L]


def _pool(pl, inp):
    """The gathered pool as every rank sees it, built without a collective."""
    parts = [S.pack_local_pages(pl, r, *_cache(inp)) for r in range(pl.world)]
    return torch.cat([p[0] for p in parts]), torch.cat([p[1] for p in parts])


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, L, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q.put(_check_rank(rank, world, L))
    except Exception as e:  # reported to the parent instead of leaving it waiting
        q.put((rank, False, repr(e)))
    finally:
        torch.distributed.destroy_process_group()


def _check_rank(rank, world, L):
    inp = W.make_inputs(_spec(L))
    pl = S.plan(L, world)
    k_local, kv_local = S.pack_local_pages(pl, rank, *_cache(inp))
    k_pool, kv_pool = S.gather_pools(k_local, kv_local)
    k_ref, kv_ref = _pool(pl, inp)
    same = bool(torch.equal(k_pool, k_ref) and torch.equal(kv_pool.view(torch.int16), kv_ref.view(torch.int16)))
    # every position's cache row, read back through the page table
    kc, ks, kv = _cache(inp)
    pt = torch.from_numpy(pl.page_table()).long()
    s = torch.arange(L)
    page, slot = pt[s // S.PAGE], s % S.PAGE
    codes = k_pool[page.unsqueeze(1), (slot * S.D_I).unsqueeze(1) + torch.arange(S.D_I)]
    sbytes = k_pool[page.unsqueeze(1), (S.PAGE * S.D_I + slot * 4).unsqueeze(1) + torch.arange(4)]
    rows = bool(torch.equal(codes, kc) and torch.equal(sbytes.contiguous().view(torch.float32).view(-1), ks)
                and torch.equal(kv_pool[page, slot].view(torch.int16), kv.view(torch.int16)))
    return rank, same, rows


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_gather_identical_pools(world):
    L = 1000
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, L, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, _, _ in res] == list(range(world))
    assert all(same for _, same, _ in res), res
    assert all(rows is True for _, _, rows in res), res


def test_oracle_on_a_rank_layout_matches_the_unsharded_sequence():
    L, world = 1000, 2
    inp = W.make_inputs(_spec(L))
    full = case_from_inputs(inp)
    pl = S.plan(L, world)
    k_pool, kv_pool = _pool(pl, inp)
    for rank in range(world):
        pos = pl.positions(rank)
        lens, cu, pt = pl.layout_arrays(rank)
        row_seq = np.repeat(np.arange(2), np.diff(cu))
        case = dict(full)
        case.update(page_size=S.PAGE, seq_lens=lens, pos=pos.astype(np.int32), row_seq=row_seq.astype(np.int32),
                    q_idx=full["q_idx"][pos], q_scale=full["q_scale"][pos], w=full["w"][pos], q=full["q"][pos],
                    k_pages=to_np(k_pool), kv=to_np(kv_pool), page_table=pt, k_idx=None, k_scale=None)
        sample = sorted({0, 1, len(pos) // 2, len(pos) - 1, int(cu[1]) - 1, int(cu[1])} & set(range(len(pos))))
        got = O.forward_rows(case, sample)
        ref = O.forward_rows(full, [int(pos[t]) for t in sample])
        for t in sample:
            g, r = got[t], ref[int(pos[t])]
            assert np.array_equal(g["scores"], r["scores"]) and np.array_equal(g["idx"], r["idx"]), (rank, t)
            assert np.array_equal(g["o"], r["o"]) and np.array_equal(g["lse"], r["lse"]), (rank, t)
