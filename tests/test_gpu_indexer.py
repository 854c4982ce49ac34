"""FP8 tcgen05 lightning indexer against the oracle (rel 1e-2 / abs 1e-3 on every
causal entry), for decode rows over contiguous and paged caches and for
prefill rows (full and partial query ranges, several sequences)."""
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


def _run(spec, rows=None):
    ensure_lib()
    inp = W.make_inputs(spec)
    case = case_from_inputs(inp)
    dc = G.to_device(inp)
    scores = G.indexer(dc)
    assert D.dsa_get_device_error() == D.DSA_OK
    sc = scores.cpu().numpy()
    rows = range(inp.T) if rows is None else rows
    ref = O.indexer_rows(case, rows)
    for t in rows:
        pos = int(case["pos"][t])
        got = sc[t, :pos + 1]
        assert not np.isnan(got).any(), (t, int(np.isnan(got).sum()))
        ok, err, nbad = indexer_close(got, ref[t])
        assert ok, (t, err, nbad)


def test_indexer_fp8_decode_contiguous():
    _run(W.DECODE_32K.replace(batch=4, lens=(5000, 129, 777, 128)))


def test_indexer_fp8_decode_paged():
    _run(W.PAGED_DECODE_128K.replace(batch=5, len_range=None, lens=(3000, 64, 1000, 65, 130)))


def test_indexer_fp8_prefill_single_sequence():
    _run(W.PREFILL_8K.replace(lens=(1000,)))


def test_indexer_fp8_prefill_partial_queries():
    # second sequence: only its last 61 tokens are queries (chunked prefill)
    spec = W.PREFILL_2X32K.replace(lens=(515, 900), q_lens=(515, 61), ar_phi=0.0)
    _run(spec)
