"""Convert generated workloads to the plain numpy dict the oracle reads."""
import numpy as np
import torch


def to_np(t):
    if t is None:
        return None
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def case_from_inputs(inp):
    s = inp.spec
    return dict(
        fp8=s.fp8, page_size=s.page_size, d_I=s.d_I, H_I=s.H_I, k=s.k, H=s.H,
        Dk=s.Dk, Dv=s.Dv, softmax_scale=s.softmax_scale,
        seq_lens=to_np(inp.seq_lens), pos=to_np(inp.pos), row_seq=to_np(inp.row_seq),
        q_idx=to_np(inp.q_idx), q_scale=to_np(inp.q_scale), k_idx=to_np(inp.k_idx),
        k_scale=to_np(inp.k_scale), k_pages=to_np(inp.k_pages), w=to_np(inp.w),
        q=to_np(inp.q), kv=to_np(inp.kv), page_table=to_np(inp.page_table))
