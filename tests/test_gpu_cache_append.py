"""Cache write (dsa_cache_append) on the GPU against the oracle, byte for byte.

Each query row's new indexer key is quantised to e4m3 with a per-token fp32 scale
and written with its latent row at the row's own position, in the paged pool
(8448-byte pages: 64 x 128 code bytes, then 64 scales) or the contiguous caches.
The whole pools are compared after the call, so a write to a wrong slot or a
stray byte fails as surely as a wrong code. The decode-loop test then scores the
appended keys with the GPU indexer and checks them against the oracle's indexer
on the oracle's appended cache."""
import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from sparse_long_context_04_b200 import device as G
from sparse_long_context_04_b200 import dsa as D
from sparse_long_context_04_b200 import workloads as W
from tests.case_utils import case_from_inputs, to_np
from tests.gpu_utils import ensure_lib, indexer_close

pytestmark = pytest.mark.gpu

PAGED = W.PAGED_DECODE_128K.replace(batch=5, len_range=None, lens=(6000, 64, 130, 4097, 1))
CONTIG = W.DECODE_32K.replace(batch=4, lens=(700, 64, 1, 2049))
PREFILL = W.PREFILL_8K.replace(lens=(300,))


def _new_tokens(T, Dk, seed, k_dtype):
    rng = np.random.default_rng(seed)
    k = (rng.standard_normal((T, 128)) * 3).astype(np.float32)
    k[0] = 0.0                                   # all-zero row: scale 1, codes 0
    if T > 2:
        k[2] *= 1e-30                            # tiny values (subnormal e4m3 codes after scaling)
        k[1, :5] = [448.0, -448.0, 1e-3, -1e-3, -0.0]
    kv = torch.from_numpy(rng.standard_normal((T, Dk)).astype(np.float32)).to(torch.bfloat16)
    kt = torch.from_numpy(k).to(k_dtype)
    k_for_oracle = kt.float().numpy()            # the values the kernel reads (bf16 rounding included)
    return kt, kv, k_for_oracle, kv.view(torch.int16).numpy().view(np.uint16)


def _append_and_compare(spec, k_dtype, seed):
    ensure_lib()
    inp = W.make_inputs(spec)
    dc = G.to_device(inp)
    case = case_from_inputs(inp)
    kt, kv, k_or, kv_or = _new_tokens(dc.T, spec.Dk, seed, k_dtype)
    paged = spec.page_size != 0
    k_scale = None if paged else dc.k_scale
    D.dsa_cache_append(kt.cuda(), kv.cuda(), dc.layout, dc.k_idx, dc.kv, k_scale)
    torch.cuda.synchronize()
    assert D.dsa_get_device_error() == D.DSA_OK
    if paged:
        k_pool0 = case["k_pages"]
        kv_pool0 = case["kv"].reshape(-1, spec.Dk)
        k_want, kv_want, _ = O.cache_append(case, k_or, kv_or, k_pool0, kv_pool0)
        s_got = s_want = None
    else:
        k_want, kv_want, s_want = O.cache_append(case, k_or, kv_or, case["k_idx"], case["kv"], case["k_scale"])
        s_got = dc.k_scale.cpu().numpy()
    k_got = dc.k_idx.cpu().numpy()
    kv_got = to_np(dc.kv.cpu()).reshape(kv_want.shape)
    assert np.array_equal(k_got, k_want), np.argwhere(k_got != k_want)[:5]
    assert np.array_equal(kv_got, kv_want)
    if s_want is not None:
        assert np.array_equal(s_got.view(np.uint32), s_want.view(np.uint32))
    return inp, dc, case, k_or, kv_or


@pytest.mark.parametrize("k_dtype", [torch.float32, torch.bfloat16])
def test_append_paged_decode_bit_exact(k_dtype):
    _append_and_compare(PAGED, k_dtype, 11)


@pytest.mark.parametrize("k_dtype", [torch.float32, torch.bfloat16])
def test_append_contiguous_decode_bit_exact(k_dtype):
    _append_and_compare(CONTIG, k_dtype, 12)


def test_append_prefill_rows_bit_exact():
    # prefill layout: every query row writes its own position (cu_q addressing)
    _append_and_compare(PREFILL, torch.float32, 13)


def test_append_then_indexer_scores_the_new_keys():
    """The decode loop: append each sequence's newest key, then score it."""
    inp, dc, case, k_or, kv_or = _append_and_compare(PAGED, torch.float32, 14)
    k_pages, kv_pool, _ = O.cache_append(case, k_or, kv_or, case["k_pages"], case["kv"].reshape(-1, PAGED.Dk))
    case2 = dict(case, k_pages=k_pages, kv=kv_pool.reshape(case["kv"].shape))
    scores = G.indexer(dc).cpu().numpy()
    ref = O.indexer_rows(case2, range(dc.T))
    for t in range(dc.T):
        n = int(case["pos"][t]) + 1
        ok, err, nbad = indexer_close(scores[t, :n], ref[t])
        assert ok, (t, err, nbad)


def test_append_reports_a_page_id_out_of_range():
    ensure_lib()
    spec = PAGED
    inp = W.make_inputs(spec)
    dc = G.to_device(inp)
    kt, kv, _, _ = _new_tokens(dc.T, spec.Dk, 15, torch.float32)
    pt = dc.layout.page_table
    b, last = 0, (int(inp.seq_lens[0]) - 1) // spec.page_size
    saved = int(pt[b, last])
    pt[b, last] = dc.layout.c.num_pages + 7      # out of the pool
    before = dc.k_idx.clone()
    D.dsa_cache_append(kt.cuda(), kv.cuda(), dc.layout, dc.k_idx, dc.kv)
    torch.cuda.synchronize()
    assert D.dsa_get_device_error() == D.DSA_ERR_DEVICE_CHECK
    pt[b, last] = saved
    # the other rows were written; nothing was written outside the pool
    assert dc.k_idx.shape == before.shape


def test_append_rejects_bad_arguments():
    ensure_lib()
    inp = W.make_inputs(PAGED)
    dc = G.to_device(inp)
    kt, kv, _, _ = _new_tokens(dc.T, PAGED.Dk, 16, torch.float32)
    with pytest.raises(D.DSAError) as ex:      # paged pools keep their scales in the pages
        D.dsa_cache_append(kt.cuda(), kv.cuda(), dc.layout, dc.k_idx, dc.kv, k_scale=torch.ones(4, device="cuda"))
    assert ex.value.status == D.DSA_ERR_INVALID_ARG
    with pytest.raises(D.DSAError) as ex:      # d_I other than 128
        D.dsa_cache_append(kt[:, :64].contiguous().cuda(), kv.cuda(), dc.layout, dc.k_idx, dc.kv)
    assert ex.value.status == D.DSA_ERR_UNSUPPORTED
