"""Move a generated workload to the GPU and call the library's stages on it.

Marshalling only (device copies, layout structs, output buffers); the stages
themselves run in libdsa.so.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

from . import dsa as D
from .workloads import Inputs


@dataclasses.dataclass
class DeviceCase:
    inp: Inputs
    q_idx: torch.Tensor
    q_scale: Optional[torch.Tensor]
    k_idx: torch.Tensor
    k_scale: Optional[torch.Tensor]
    w: torch.Tensor
    q: torch.Tensor
    kv: torch.Tensor
    layout: D.Layout
    ld: int

    @property
    def T(self) -> int:
        return int(self.q.shape[0])


def to_device(inp: Inputs, device="cuda") -> DeviceCase:
    s = inp.spec
    dev = torch.device(device)
    seq_lens = inp.seq_lens.to(dev)
    cu_q = None if inp.cu_q is None else inp.cu_q.to(dev)
    if s.page_size:
        page_table = inp.page_table.to(dev)
        k_idx = inp.k_pages.to(dev)
        k_scale = None
        layout = D.Layout(seq_lens, inp.n_max, cu_q, page_table, s.page_size, int(inp.k_pages.shape[0]))
    else:
        k_idx = inp.k_idx.to(dev)
        k_scale = None if inp.k_scale is None else inp.k_scale.to(dev)
        layout = D.Layout(seq_lens, inp.n_max, cu_q)
    ld = (layout.capacity + 3) // 4 * 4
    return DeviceCase(
        inp=inp, q_idx=inp.q_idx.to(dev), q_scale=None if inp.q_scale is None else inp.q_scale.to(dev),
        k_idx=k_idx, k_scale=k_scale, w=inp.w.to(dev), q=inp.q.to(dev), kv=inp.kv.to(dev), layout=layout, ld=ld)


def indexer(dc: DeviceCase, scores: Optional[torch.Tensor] = None) -> torch.Tensor:
    if scores is None:
        scores = torch.full((dc.T, dc.ld), float("nan"), dtype=torch.float32, device=dc.q.device)
    D.dsa_indexer_scores(dc.q_idx, dc.q_scale, dc.k_idx, dc.k_scale, dc.w, dc.layout, scores)
    return scores


def topk(dc: DeviceCase, scores: torch.Tensor, idx: Optional[torch.Tensor] = None) -> torch.Tensor:
    if idx is None:
        idx = torch.empty((dc.T, dc.inp.spec.k), dtype=torch.int32, device=scores.device)
    D.dsa_topk(scores, dc.inp.spec.k, dc.layout, idx)
    return idx


def attention(dc: DeviceCase, idx: torch.Tensor, out=None, lse=None, workspace=None):
    s = dc.inp.spec
    if out is None:
        out = torch.empty((dc.T, s.H, s.Dv), dtype=dc.q.dtype, device=dc.q.device)
    if lse is None:
        lse = torch.empty((dc.T, s.H), dtype=torch.float32, device=dc.q.device)
    if workspace is None:
        n = D.dsa_sparse_mqa_attn_workspace_size(dc.T, s.H, s.Dv, int(idx.shape[1]), dc.q)
        workspace = torch.empty(max(n, 1), dtype=torch.uint8, device=dc.q.device)
    D.dsa_sparse_mqa_attn(dc.q, dc.kv, idx, dc.layout, out, lse, s.softmax_scale, workspace)
    return out, lse


def indexer_kl(dc: DeviceCase, idx: torch.Tensor, lse: torch.Tensor, scores: torch.Tensor, loss=None, grad=None,
               want_grad=True):
    if loss is None:
        loss = torch.empty(dc.T, dtype=torch.float32, device=dc.q.device)
    if grad is None and want_grad:
        grad = torch.empty(tuple(idx.shape), dtype=torch.float32, device=dc.q.device)
    D.dsa_indexer_kl(dc.q, dc.kv, idx, dc.layout, lse, scores, loss, dc.inp.spec.softmax_scale, grad)
    return loss, grad


class Forward:
    """dsa_forward with its buffers allocated once (reusable across steps)."""

    def __init__(self, dc: DeviceCase, keep_idx: bool = True, topk_path: int = D.DSA_TOPK_AUTO,
                 out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None):
        s = dc.inp.spec
        dev = dc.q.device
        self.dc = dc
        self.out = torch.empty((dc.T, s.H, s.Dv), dtype=dc.q.dtype, device=dev) if out is None else out
        self.lse = torch.empty((dc.T, s.H), dtype=torch.float32, device=dev) if lse is None else lse
        self.idx = torch.empty((dc.T, s.k), dtype=torch.int32, device=dev) if keep_idx else None
        self.args = D.forward_args(dc.q_idx, dc.q_scale, dc.k_idx, dc.k_scale, dc.w, dc.q, dc.kv, s.k,
                                   s.softmax_scale, dc.layout, self.out, self.lse, self.idx, topk_path)
        n = D.dsa_forward_workspace_size(self.args)
        if n == 0:
            raise D.DSAError(D.DSA_ERR_INVALID_ARG, "dsa_forward_workspace_size")
        self.workspace = torch.empty(n, dtype=torch.uint8, device=dev)

    def __call__(self, stream=None):
        D.dsa_forward(self.args, self.workspace, stream)
        return self.out, self.lse, self.idx
