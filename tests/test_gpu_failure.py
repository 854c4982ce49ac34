"""Failure detection without faulting the GPU: every on-device wait is bounded.
With the bound set to 1 ns the kernels' waits run out; the kernels record
DSA_ERR_TIMEOUT (and the failing wait's site) in the device error word and wind
down cleanly. Afterwards the same context computes correct results again.
Also: a page id outside the pool is caught by the device bounds check."""
import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from sparse_long_context_04_b200 import device as G
from sparse_long_context_04_b200 import dsa as D
from sparse_long_context_04_b200 import workloads as W
from tests.case_utils import case_from_inputs
from tests.gpu_utils import ensure_lib, indexer_close

pytestmark = pytest.mark.gpu


def _spec():
    return W.PAGED_DECODE_128K.replace(batch=3, len_range=None, lens=(9000, 5000, 2049))


def test_bounded_waits_time_out_and_the_context_recovers():
    ensure_lib()
    inp = W.make_inputs(_spec())
    case = case_from_inputs(inp)
    dc = G.to_device(inp)
    D.dsa_get_device_error()          # start from a clean error word
    try:
        D.dsa_set_wait_limit_ns(1)
        fw = G.Forward(dc)
        fw()
        st, site = D.dsa_get_device_error_site()
        assert st == D.DSA_ERR_TIMEOUT, st
        assert site != 0
        assert D.dsa_get_device_error() == D.DSA_OK   # read and cleared
    finally:
        D.dsa_set_wait_limit_ns(1_000_000_000)
    torch.cuda.synchronize()
    # the context is still usable and the results are right
    out, lse, idx = G.Forward(dc)()
    assert D.dsa_get_device_error() == D.DSA_OK
    scores = G.indexer(dc).cpu().numpy()
    ref = O.indexer_rows(case, range(3))
    for t in range(3):
        pos = int(case["pos"][t])
        assert indexer_close(scores[t, :pos + 1], ref[t])[0]
        assert np.array_equal(idx[t].cpu().numpy(), O.topk_row(scores[t, :pos + 1], 2048))


def test_page_id_outside_the_pool_is_reported():
    ensure_lib()
    inp = W.make_inputs(_spec())
    dc = G.to_device(inp)
    D.dsa_get_device_error()
    dc.layout.page_table[1, 3] = dc.layout.c.num_pages + 5   # corrupt one entry of sequence 1
    G.indexer(dc)
    st, site = D.dsa_get_device_error_site()
    assert st == D.DSA_ERR_DEVICE_CHECK and site != 0
