"""Prefill of one long sequence on several GPUs, one process per GPU.

A query row at position p scores and attends over p + 1 keys, so equal
consecutive ranges of rows would leave the last rank with most of the work.
Instead the sequence is cut into 2 * world chunks of C tokens (C a multiple of
the 64-token cache page) and rank r takes chunks r and 2 * world - 1 - r: chunk i
costs about (i + 1/2) C^2 key visits, so every rank's pair costs the same.

Every rank needs the whole prefix's indexer keys and latent rows. Each rank
holds the cache pages of its own two chunks (the paged formats of the C ABI: an
8448-byte indexer-key page of 64 x 128 e4m3 codes followed by 64 fp32 scales, and
a 64 x 576 bf16 latent page); one all-gather copies every rank's pages into a
pool in local memory, and a page table, computed on the host, maps the
sequence's logical pages into that pool. No other data moves. The rank's query
rows then run as a two-piece prefill (one piece per chunk, rows in chunk order)
over the same page table: piece j holds the rows of chunk c_j and its sequence
length is the chunk's end, so each row's causal range is unchanged.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch
import torch.distributed as dist

PAGE = 64
D_I = 128
K_PAGE_BYTES = PAGE * D_I + 4 * PAGE   # 8448


@dataclasses.dataclass(frozen=True)
class ShardPlan:
    L: int              # tokens in the sequence
    world: int
    C: int              # tokens per chunk, a multiple of PAGE

    @property
    def n_chunks(self) -> int:
        return 2 * self.world

    @property
    def pages_per_chunk(self) -> int:
        return self.C // PAGE

    @property
    def max_pages(self) -> int:
        """Logical pages of the sequence."""
        return -(-self.L // PAGE)

    @property
    def pool_pages(self) -> int:
        """Pages in the gathered pool (every rank contributes two chunks)."""
        return self.world * 2 * self.pages_per_chunk

    def chunks(self, rank: int):
        """The two chunk ids of `rank`, in the order its rows are laid out."""
        return rank, self.n_chunks - 1 - rank

    def chunk_rows(self, chunk: int):
        """[start, stop) token positions of a chunk (empty past the sequence end)."""
        a = min(self.L, chunk * self.C)
        return a, min(self.L, (chunk + 1) * self.C)

    def positions(self, rank: int) -> np.ndarray:
        """Positions of the rank's query rows, in row order."""
        return np.concatenate([np.arange(*self.chunk_rows(c)) for c in self.chunks(rank)]).astype(np.int64)

    def cost(self, rank: int) -> int:
        """Key visits of the rank's rows under causal attention: sum of (pos + 1)."""
        return int((self.positions(rank) + 1).sum())

    def page_table(self) -> np.ndarray:
        """int32 [max_pages]: the pool page holding each logical page."""
        out = np.empty(self.max_pages, dtype=np.int32)
        ppc = self.pages_per_chunk
        for p in range(self.max_pages):
            c, o = divmod(p, ppc)
            owner = c if c < self.world else self.n_chunks - 1 - c
            slot = 0 if c < self.world else 1
            out[p] = (owner * 2 + slot) * ppc + o
        return out

    def layout_arrays(self, rank: int):
        """(seq_lens int32 [2], cu_q int32 [3], page_table int32 [2][max_pages]) of the
        rank's two-piece prefill, for a paged dsa_seq_layout with num_pages =
        pool_pages and n_max = L."""
        lens, cu = [], [0]
        for c in self.chunks(rank):
            a, b = self.chunk_rows(c)
            lens.append(max(b, 1))          # an empty chunk past the end keeps a valid length
            cu.append(cu[-1] + (b - a))
        pt = np.stack([self.page_table()] * 2)
        return np.array(lens, np.int32), np.array(cu, np.int32), pt


def plan(L: int, world: int) -> ShardPlan:
    """Chunks of the smallest page multiple that covers L in 2 * world chunks."""
    if L < 1 or world < 1:
        raise ValueError("need L >= 1 and world >= 1")
    per = -(-L // (2 * world))
    return ShardPlan(L=L, world=world, C=-(-per // PAGE) * PAGE)


def pack_local_pages(pl: ShardPlan, rank: int, k_codes: torch.Tensor, k_scale: torch.Tensor, kv: torch.Tensor):
    """The rank's own pages from its tokens' cache rows.

    k_codes uint8 [L][128], k_scale float32 [L], kv bf16 [L][Dk] hold the whole
    sequence by position (only the rank's chunks are read). Returns the indexer-key
    pages uint8 [2 * pages_per_chunk][8448] and the latent pages bf16
    [2 * pages_per_chunk][64][Dk], chunk by chunk in the rank's order; slots past
    the sequence end are zero codes with scale 1 and zero rows."""
    ppc, Dk = pl.pages_per_chunk, int(kv.shape[1])
    kp = torch.zeros((2 * ppc, PAGE, D_I), dtype=torch.uint8, device=k_codes.device)
    sp = torch.ones((2 * ppc, PAGE), dtype=torch.float32, device=k_codes.device)
    vp = torch.zeros((2 * ppc, PAGE, Dk), dtype=kv.dtype, device=kv.device)
    for j, c in enumerate(pl.chunks(rank)):
        a, b = pl.chunk_rows(c)
        n = b - a
        if n <= 0:
            continue
        dst = slice(j * ppc * PAGE, j * ppc * PAGE + n)
        kp.view(-1, D_I)[dst] = k_codes[a:b]
        sp.view(-1)[dst] = k_scale[a:b]
        vp.view(-1, Dk)[dst] = kv[a:b]
    k_pages = torch.cat([kp.view(2 * ppc, -1), sp.view(torch.uint8).view(2 * ppc, -1)], dim=1).contiguous()
    return k_pages, vp


def gather_pools(k_local: torch.Tensor, kv_local: torch.Tensor, group=None):
    """All ranks' pages into one pool in local memory, rank by rank (the pool page
    numbering that ShardPlan.page_table assumes). One all-gather per cache."""
    world = dist.get_world_size(group)

    def gather(x):
        bits = x.view(torch.uint8)          # bytes: every backend carries them
        if dist.get_backend(group) == "nccl":
            out = torch.empty((world * bits.shape[0],) + tuple(bits.shape[1:]), dtype=bits.dtype, device=bits.device)
            dist.all_gather_into_tensor(out, bits.contiguous(), group=group)
        else:
            parts = [torch.empty_like(bits) for _ in range(world)]
            dist.all_gather(parts, bits.contiguous(), group=group)
            out = torch.cat(parts)
        return out.view(x.dtype)

    return gather(k_local), gather(kv_local)
