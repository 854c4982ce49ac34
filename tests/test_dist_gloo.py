"""The multi-process host path on CPU: two gloo ranks agree on the slowest rank's
time, get different seeds for their batches, and compute the whole-job rate."""
import os
import socket

import torch.multiprocessing as mp

from sparse_long_context_04_b200 import dist as X


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    X.init("gloo", timeout_s=60)
    w, r, lr = X.rank_info()
    mx = X.max_over_ranks(10.0 + 5.0 * rank)      # rank 1 is the slower one
    seed = X.rank_seed(0xD5A0, rank)
    rate = X.job_rate(w, 16, 100, mx)
    X.barrier()
    X.finish()
    q.put((r, w, mx, seed, rate))


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, m0, s0, v0), (r1, w1, m1, s1, v1) = res
    assert (r0, r1) == (0, 1) and w0 == w1 == 2
    assert m0 == m1 == 15.0                        # max over ranks, seen by both
    assert s0 != s1
    assert abs(v0 - 2 * 16 * 100 / 0.015) < 1e-6 and v0 == v1


def test_single_process_defaults():
    assert X.rank_info()[0] >= 1
    assert X.max_over_ranks(3.5) == 3.5
    assert X.job_rate(1, 16, 10, 1.0) == 160000.0
