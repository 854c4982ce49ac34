"""The seeded input generator: determinism, shapes, layouts and planted structure."""
import numpy as np
import torch

from sparse_long_context_04_b200 import workloads as W


def test_deterministic_and_shaped():
    spec = W.PAGED_DECODE_128K.replace(batch=2, len_range=None, lens=(130, 64))
    a, b = W.make_inputs(spec), W.make_inputs(spec)
    for f in ("q_idx", "q_scale", "k_pages", "w", "q", "kv", "page_table"):
        assert torch.equal(getattr(a, f), getattr(b, f)), f
    assert a.k_pages.shape == (3 + 1, 64 * 128 + 4 * 64)
    assert a.kv.shape == (4, 64, 576) and a.kv.dtype == torch.bfloat16
    assert a.page_table.shape == (2, 3)
    # one global permutation dealt in order: every physical page used once
    used = torch.cat([a.page_table[0, :3], a.page_table[1, :1]])
    assert sorted(used.tolist()) == [0, 1, 2, 3]
    assert a.pos.tolist() == [129, 63] and a.cu_q is None


def test_prefill_rows_and_lengths():
    spec = W.TINY
    x = W.make_inputs(spec)
    assert x.T == 256 and x.cu_q.tolist() == [0, 256]
    assert x.pos.tolist() == list(range(256))
    assert x.q_idx.dtype == torch.float32 and x.kv.shape == (1, 256, 64)


def test_drawn_lengths_in_range():
    lens = W.draw_lens(W.PAGED_DECODE_128K)
    assert len(lens) == 16 and all(98304 <= L <= 131072 for L in lens)


def test_planted_keys_correlate_with_query():
    spec = W.DECODE_32K.replace(batch=2, lens=(4000, 4000))
    x = W.make_inputs(spec)
    kv = x.kv[0, :4000].float()
    q0 = x.q[0, 0].float()
    cos = (kv @ q0) / (kv.norm(dim=1) * q0.norm())
    # 1% planted rows with rho = 0.8 stand far above the iid bulk
    assert int((cos > 0.5).sum()) == 40


def test_ar1_keys_are_locally_correlated():
    spec = W.PREFILL_2X32K.replace(lens=(2000, 1000), fp8=True)
    x = W.make_inputs(spec)
    k = x.kv[0, :2000].float()
    c1 = torch.nn.functional.cosine_similarity(k[1:], k[:-1]).mean().item()
    assert 0.85 < c1 < 0.95
