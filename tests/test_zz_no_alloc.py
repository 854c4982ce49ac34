"""The attention entry point that allocates nothing (dsa_sparse_mqa_attn_noalloc).

It serves callers that may not allocate device memory — code under a host
framework that has reserved all device memory up front, or a serving loop that
cannot afford cudaMalloc's implicit synchronisation. Its split partials live in
the library's own 40 MiB static device array instead of a caller workspace.
Both entry points run the same kernels on the same split plan, so their outputs
must be identical bit for bit: on two calls in a row, and at the array's
capacity (39 decode rows at k = 2048) right after a call on other inputs, so
that anything read from a previous call's scratch would show. A call that does
not fit the array must be refused before anything is launched.
"""
import pytest
import torch

from sparse_long_context_04_b200 import device as G
from sparse_long_context_04_b200 import dsa as D
from sparse_long_context_04_b200 import workloads as W
from tests.gpu_utils import ensure_lib

pytestmark = pytest.mark.gpu


def _reference(dc):
    idx = G.topk(dc, G.indexer(dc))
    out, lse = G.attention(dc, idx)
    torch.cuda.synchronize()
    assert D.dsa_get_device_error() == D.DSA_OK
    return idx, out, lse


def _noalloc(dc, idx, like_out, like_lse):
    out = torch.full_like(like_out, float("nan"))
    lse = torch.full_like(like_lse, float("nan"))
    D.dsa_sparse_mqa_attn_noalloc(dc.q, dc.kv, idx, dc.layout, out, lse, dc.inp.spec.softmax_scale)
    torch.cuda.synchronize()
    assert D.dsa_get_device_error() == D.DSA_OK
    return out, lse


def _same(a, b):
    return torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a,
                       b.view(torch.int16) if b.dtype == torch.bfloat16 else b)


def test_noalloc_matches_workspace_entry_point_twice():
    ensure_lib()
    spec = W.PAGED_DECODE_128K.replace(batch=5, len_range=None, lens=(6000, 2048, 300, 4097, 64))
    dc = G.to_device(W.make_inputs(spec))
    idx, ref_out, ref_lse = _reference(dc)
    for _ in range(2):
        out, lse = _noalloc(dc, idx, ref_out, ref_lse)
        assert _same(out, ref_out) and _same(lse, ref_lse)


def test_noalloc_at_capacity_after_a_call_on_other_inputs():
    ensure_lib()
    base = W.PAGED_DECODE_128K.replace(batch=39, len_range=(2100, 6000))
    dc_a = G.to_device(W.make_inputs(base))
    dc_b = G.to_device(W.make_inputs(base.replace(seed=base.seed + 100)))
    idx_a, out_a, lse_a = _reference(dc_a)
    idx_b, out_b, lse_b = _reference(dc_b)
    got_a = _noalloc(dc_a, idx_a, out_a, lse_a)      # fills the whole array with case A's partials
    got_b = _noalloc(dc_b, idx_b, out_b, lse_b)
    assert _same(got_a[0], out_a) and _same(got_a[1], lse_a)
    assert _same(got_b[0], out_b) and _same(got_b[1], lse_b)


def test_noalloc_rejects_calls_beyond_its_scratch():
    ensure_lib()
    # 40 decode rows x 8 splits of 2048 selected positions need 40.3 MiB of partials
    spec = W.DECODE_32K.replace(batch=40, lens=(64,) * 40)
    dc = G.to_device(W.make_inputs(spec))
    idx = torch.full((40, spec.k), -1, dtype=torch.int32, device="cuda")
    out = torch.zeros((40, spec.H, spec.Dv), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((40, spec.H), dtype=torch.float32, device="cuda")
    with pytest.raises(D.DSAError) as ex:
        D.dsa_sparse_mqa_attn_noalloc(dc.q, dc.kv, idx, dc.layout, out, lse, spec.softmax_scale)
    assert ex.value.status == D.DSA_ERR_TOO_LARGE
    torch.cuda.synchronize()
    assert out.abs().max().item() == 0      # nothing was launched
