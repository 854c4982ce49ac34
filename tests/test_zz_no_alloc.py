"""The attention entry point that allocates nothing (dsa_sparse_mqa_attn_noalloc).

It serves callers that may not allocate device memory — code under a host
framework that has reserved all device memory up front, or a serving loop that
cannot afford cudaMalloc's implicit synchronisation. Its split partials live in
the library's own 40 MiB static device array instead of a caller workspace.
Called twice in a row through the C ABI, it must give the same output as the
workspace entry point, and it must refuse a call that would not fit the array.
"""
import numpy as np
import pytest
import torch

from sparse_long_context_04_b200 import device as G
from sparse_long_context_04_b200 import dsa as D
from sparse_long_context_04_b200 import workloads as W
from tests.gpu_utils import ensure_lib

pytestmark = pytest.mark.gpu
TOL = 2e-2   # the attention tolerance used by the other bf16 parity tests


def test_noalloc_matches_workspace_entry_point_twice():
    ensure_lib()
    spec = W.PAGED_DECODE_128K.replace(batch=5, len_range=None, lens=(6000, 2048, 300, 4097, 64))
    inp = W.make_inputs(spec)
    dc = G.to_device(inp)
    idx = G.topk(dc, G.indexer(dc))
    ref_out, ref_lse = G.attention(dc, idx)
    torch.cuda.synchronize()
    assert D.dsa_get_device_error() == D.DSA_OK
    for _ in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        D.dsa_sparse_mqa_attn_noalloc(dc.q, dc.kv, idx, dc.layout, out, lse, spec.softmax_scale)
        torch.cuda.synchronize()
        assert D.dsa_get_device_error() == D.DSA_OK
        e_out = (out.float() - ref_out.float()).abs().max().item()
        e_lse = (lse - ref_lse).abs().max().item()
        assert e_out <= TOL and e_lse <= TOL, (e_out, e_lse)


def test_noalloc_rejects_calls_beyond_its_scratch():
    ensure_lib()
    # 48 decode rows x 8 splits of 2048 selected positions need 48 MiB of partials
    spec = W.DECODE_32K.replace(batch=48, lens=(64,) * 48)
    inp = W.make_inputs(spec)
    dc = G.to_device(inp)
    idx = torch.full((48, spec.k), -1, dtype=torch.int32, device="cuda")
    out = torch.zeros((48, spec.H, spec.Dv), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((48, spec.H), dtype=torch.float32, device="cuda")
    with pytest.raises(D.DSAError) as ex:
        D.dsa_sparse_mqa_attn_noalloc(dc.q, dc.kv, idx, dc.layout, out, lse, spec.softmax_scale)
    assert ex.value.status == D.DSA_ERR_TOO_LARGE
    torch.cuda.synchronize()
    assert out.abs().max().item() == 0      # nothing was launched
