"""Seeded synthetic workloads for the DSA hot path.

This module only *makes inputs*: shapes, seeded random values, planted
structure, FP8/bf16 encoding and the paged layout. It computes none of the
method's arithmetic (no indexer scores, no selection, no attention), so both the
CUDA path and the CPU oracle can consume what it produces.

Workloads follow the DeepSeek-V3.2-Exp pages ("DeepSeek-V3.2-Exp" on jdon.com:
k = 2048 selected tokens, FP8 indexer with few heads, 128K context; mundobytes
run guide: page size 64 for the KV cache). Head shapes (H_I = 64, d_I = 128,
128 query heads over a 576-wide latent row whose first 512 dims are the value)
are the configuration this library is built for.

Layouts produced (torch CPU tensors, row-major):
  FP8 indexer:  q_idx  uint8  [T, H_I, d_I]  (e4m3 bytes),  q_scale f32 [T]
                k_idx  uint8  [B, N, d_I],   k_scale f32 [B, N]     (contiguous)
                k_pages uint8 [P, page*d_I + page*4]                 (paged: keys, then fp32 scales)
  fp32 indexer: q_idx  f32 [T, H_I, d_I], k_idx f32 [B, N, d_I], no scales
  weights:      w f32 [T, H_I]
  attention:    q  bf16 [T, H, Dk];  kv bf16 [B, N, Dk] (contiguous) or [P, page, Dk] (paged)
                (fp32 in the fp32 workload)
  addressing:   seq_lens int32 [B]; cu_q int32 [B+1] (prefill) or None (decode);
                page_table int32 [B, max_pages] (paged) or None
Query row t of sequence b sits at position pos = len_b - q_len_b + i (the
last q_len_b tokens of the sequence); in decode q_len_b = 1, pos = len_b - 1.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import math
import os
import zlib
from typing import Optional

import numpy as np
import torch

E4M3_MAX = 448.0


@dataclasses.dataclass(frozen=True)
class Spec:
    name: str
    mode: str                      # "prefill" | "decode"
    batch: int
    lens: Optional[tuple] = None   # fixed per-sequence key counts
    len_range: Optional[tuple] = None  # (lo, hi) inclusive: lengths drawn uniformly
    q_lens: Optional[tuple] = None     # prefill: query rows per sequence (default: all)
    H_I: int = 64
    d_I: int = 128
    k: int = 2048
    H: int = 128
    Dk: int = 576
    Dv: int = 512
    softmax_scale: float = 1.0 / math.sqrt(192.0)
    fp8: bool = True
    page_size: int = 0
    w_std: float = 1.0 / 8.0
    plant: str = "none"            # "none" | "tiny" | "frac"
    plant_frac: float = 0.0
    plant_count: int = 8
    ar_phi: float = 0.0
    seed: int = 0xD5A0

    def replace(self, **kw) -> "Spec":
        return dataclasses.replace(self, **kw)


# The five workloads, in the order the method's configurations are listed.
TINY = Spec(
    name="tiny_fp32_prefill_L256", mode="prefill", batch=1, lens=(256,),
    H_I=4, d_I=32, k=64, H=8, Dk=64, Dv=32, softmax_scale=1.0 / 8.0, fp8=False,
    w_std=0.5, plant="tiny", plant_count=8, seed=0xD5A0 + 1)
DECODE_32K = Spec(
    name="decode_b32_ctx32k", mode="decode", batch=32, lens=(32768,) * 32,
    plant="frac", plant_frac=0.01, seed=0xD5A0 + 2)
PREFILL_8K = Spec(
    name="prefill_L8192", mode="prefill", batch=1, lens=(8192,), seed=0xD5A0 + 3)
PREFILL_2X32K = Spec(
    name="prefill_2x32768_ar1", mode="prefill", batch=2, lens=(32768, 32768),
    ar_phi=0.9, seed=0xD5A0 + 4)
PAGED_DECODE_128K = Spec(
    name="paged_decode_b16_ctx96k_128k", mode="decode", batch=16,
    len_range=(98304, 131072), page_size=64, plant="frac", plant_frac=0.005,
    seed=0xD5A0 + 5)

WORKLOADS = {s.name: s for s in (TINY, DECODE_32K, PREFILL_8K, PREFILL_2X32K, PAGED_DECODE_128K)}


@dataclasses.dataclass
class Inputs:
    spec: Spec
    seq_lens: torch.Tensor            # int32 [B]
    cu_q: Optional[torch.Tensor]      # int32 [B+1] or None (decode)
    pos: torch.Tensor                 # int32 [T]: position of each query row
    row_seq: torch.Tensor             # int32 [T]: sequence of each query row
    q_idx: torch.Tensor
    q_scale: Optional[torch.Tensor]
    k_idx: Optional[torch.Tensor]     # contiguous indexer keys
    k_scale: Optional[torch.Tensor]
    k_pages: Optional[torch.Tensor]   # paged indexer keys + scales
    w: torch.Tensor
    q: torch.Tensor
    kv: torch.Tensor                  # [B, N, Dk] or [P, page, Dk]
    page_table: Optional[torch.Tensor]
    n_max: int

    @property
    def T(self) -> int:
        return int(self.pos.numel())


# --------------------------------------------------------------------------
# seeded streams

def _rng(seed: int, *names) -> np.random.Generator:
    key = [seed & 0xFFFFFFFF] + [zlib.crc32(str(n).encode()) for n in names]
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(key)))


_CHUNK_ROWS = 4096


def _normal(seed, name, shape, chunk_rows=_CHUNK_ROWS, threads=None) -> np.ndarray:
    """N(0,1) float32 array of `shape`, generated in row chunks from independent streams."""
    shape = tuple(int(x) for x in shape)
    out = np.empty(shape, dtype=np.float32)
    if out.size == 0:
        return out
    rows = shape[0]
    flat = out.reshape(rows, -1)
    chunks = [(r, min(rows, r + chunk_rows)) for r in range(0, rows, chunk_rows)]

    def fill(c):
        r0, r1 = c
        g = _rng(seed, name, r0)
        flat[r0:r1] = g.standard_normal((r1 - r0, flat.shape[1]), dtype=np.float32)

    threads = threads or min(16, os.cpu_count() or 1)
    if len(chunks) == 1 or threads == 1:
        for c in chunks:
            fill(c)
    else:
        with _cf.ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, chunks))
    return out


def _ar1(x: np.ndarray, phi: float) -> np.ndarray:
    """In place: x[s] <- phi*x[s-1] + sqrt(1-phi^2)*z[s] along axis 0 (x[0] = z[0])."""
    c = np.float32(math.sqrt(1.0 - phi * phi))
    p = np.float32(phi)
    for s in range(1, x.shape[0]):
        x[s] = p * x[s - 1] + c * x[s]
    return x


# --------------------------------------------------------------------------
# encoders (input preparation: both sides then read identical bytes)

def encode_e4m3_per_token(x: np.ndarray):
    """Per-token (leading axis) e4m3 quantisation: scale = max|x| / 448, bytes = RNE(x / scale)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    lead = t.shape[0]
    flat = t.reshape(lead, -1)
    amax = flat.abs().amax(dim=1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = (flat / scale[:, None]).clamp_(-E4M3_MAX, E4M3_MAX)
    q8 = y.to(torch.float8_e4m3fn).view(torch.uint8).reshape(t.shape)
    return q8, scale.to(torch.float32)


def encode_bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


# --------------------------------------------------------------------------

def draw_lens(spec: Spec) -> list:
    if spec.lens is not None:
        assert len(spec.lens) == spec.batch
        return [int(x) for x in spec.lens]
    lo, hi = spec.len_range
    g = _rng(spec.seed, "lens")
    return [int(v) for v in g.integers(lo, hi + 1, size=spec.batch)]


def make_inputs(spec: Spec, big_q_device=None) -> Inputs:
    """Build every input tensor of `spec` on the host (torch CPU tensors).

    big_q_device: for the large prefill workloads, whose iid query block is
    gigabytes, draw that block directly on this device (torch's generator, seeded
    from the workload seed; N(0,1) rounded to bf16) instead of on the host. Used by
    the benchmark only; its values differ from the host stream's."""
    lens = draw_lens(spec)
    B = spec.batch
    if spec.mode == "decode":
        q_lens = [1] * B
    else:
        q_lens = list(spec.q_lens) if spec.q_lens is not None else list(lens)
    assert all(1 <= ql <= L for ql, L in zip(q_lens, lens))
    T = sum(q_lens)
    n_max = max(lens)
    seed = spec.seed

    pos = np.concatenate([np.arange(L - ql, L, dtype=np.int32) for ql, L in zip(q_lens, lens)])
    row_seq = np.concatenate([np.full(ql, b, dtype=np.int32) for b, ql in enumerate(q_lens)])
    cu_q = None
    if spec.mode == "prefill":
        cu_q = torch.tensor(np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32))

    # ---- query side (iid) ----
    qI = _normal(seed, "q_idx", (T, spec.H_I, spec.d_I))
    w = _normal(seed, "w", (T, spec.H_I)) * np.float32(spec.w_std)
    big_q = spec.plant != "frac" and T * spec.H * spec.Dk > (1 << 28)
    # large prefill queries are generated and encoded chunk by chunk (same values)
    q = None if big_q else _normal(seed, "q", (T, spec.H, spec.Dk))

    # ---- key side, per sequence in logical order ----
    kI_seq, kv_seq = [], []
    for b, L in enumerate(lens):
        kI = _normal(seed, f"k_idx/{b}", (L, spec.d_I))
        kv = _normal(seed, f"kv/{b}", (L, spec.Dk))
        if spec.ar_phi:
            _ar1(kI, spec.ar_phi)
            _ar1(kv, spec.ar_phi)
        kI_seq.append(kI)
        kv_seq.append(kv)

    # ---- planted high-similarity keys ----
    if spec.plant == "tiny":
        g = _rng(seed, "plant")
        L = lens[0]
        ps = g.choice(L, size=spec.plant_count, replace=False)
        for p in ps:
            t = int(g.integers(p, L))
            j = int(np.argmax(w[t]))
            z = g.standard_normal(spec.d_I).astype(np.float32)
            kI_seq[0][p] = 0.8 * qI[t, j] + 0.6 * z
    elif spec.plant == "frac":
        assert spec.mode == "decode"
        for b, L in enumerate(lens):
            g = _rng(seed, "plant", b)
            n = int(round(spec.plant_frac * L))
            ps = g.choice(L, size=n, replace=False)
            j = int(np.argmax(w[b]))
            zk = g.standard_normal((n, spec.d_I)).astype(np.float32)
            zv = g.standard_normal((n, spec.Dk)).astype(np.float32)
            kI_seq[b][ps] = 0.8 * qI[b, j][None, :] + 0.6 * zk
            kv_seq[b][ps] = 0.8 * q[b, 0][None, :] + 0.6 * zv

    # ---- encode ----
    if spec.fp8:
        q_idx, q_scale = encode_e4m3_per_token(qI)
        if big_q and big_q_device is not None:
            g = torch.Generator(device=big_q_device).manual_seed(zlib.crc32(b"q") ^ (seed & 0xFFFFFFFF))
            q_t = torch.randn((T, spec.H, spec.Dk), generator=g, device=big_q_device,
                              dtype=torch.float32).to(torch.bfloat16)
        elif big_q:
            q_t = torch.empty((T, spec.H, spec.Dk), dtype=torch.bfloat16)
            for r0 in range(0, T, _CHUNK_ROWS):
                r1 = min(T, r0 + _CHUNK_ROWS)
                g = _rng(seed, "q", r0)
                q_t[r0:r1] = encode_bf16(g.standard_normal((r1 - r0, spec.H, spec.Dk), dtype=np.float32))
        else:
            q_t = encode_bf16(q)
    else:
        q_idx, q_scale = torch.from_numpy(qI), None
        q_t = torch.from_numpy(q)
    w_t = torch.from_numpy(np.ascontiguousarray(w))

    page_table = None
    k_idx = k_scale = k_pages = None
    P = spec.page_size
    if P == 0:
        if spec.fp8:
            k_idx = torch.zeros((B, n_max, spec.d_I), dtype=torch.uint8)
            k_scale = torch.ones((B, n_max), dtype=torch.float32)
            kv_t = torch.zeros((B, n_max, spec.Dk), dtype=torch.bfloat16)
        else:
            k_idx = torch.zeros((B, n_max, spec.d_I), dtype=torch.float32)
            kv_t = torch.zeros((B, n_max, spec.Dk), dtype=torch.float32)
        for b, L in enumerate(lens):
            if spec.fp8:
                k8, ks = encode_e4m3_per_token(kI_seq[b])
                k_idx[b, :L] = k8
                k_scale[b, :L] = ks
                kv_t[b, :L] = encode_bf16(kv_seq[b])
            else:
                k_idx[b, :L] = torch.from_numpy(kI_seq[b])
                kv_t[b, :L] = torch.from_numpy(kv_seq[b])
    else:
        assert spec.fp8, "paged layout is defined for the FP8 indexer cache"
        npages = [(L + P - 1) // P for L in lens]
        total = sum(npages)
        max_pages = max(npages)
        perm = _rng(seed, "pages").permutation(total).astype(np.int32)
        pt = np.zeros((B, max_pages), dtype=np.int32)
        off = 0
        for b, n in enumerate(npages):
            pt[b, :n] = perm[off:off + n]
            off += n
        page_table = torch.from_numpy(pt)
        kb = P * spec.d_I
        k_pages = torch.zeros((total, kb + 4 * P), dtype=torch.uint8)
        kv_t = torch.zeros((total, P, spec.Dk), dtype=torch.bfloat16)
        for b, L in enumerate(lens):
            n = npages[b]
            k8, ks = encode_e4m3_per_token(kI_seq[b])
            kpad = torch.zeros((n * P, spec.d_I), dtype=torch.uint8)
            kpad[:L] = k8
            spad = torch.ones((n * P,), dtype=torch.float32)
            spad[:L] = ks
            vpad = torch.zeros((n * P, spec.Dk), dtype=torch.bfloat16)
            vpad[:L] = encode_bf16(kv_seq[b])
            ids = torch.from_numpy(pt[b, :n].astype(np.int64))
            k_pages[ids, :kb] = kpad.reshape(n, kb)
            k_pages[ids, kb:] = spad.reshape(n, P).contiguous().view(torch.uint8).reshape(n, 4 * P)
            kv_t[ids] = vpad.reshape(n, P, spec.Dk)
        kI_seq = kv_seq = None

    return Inputs(
        spec=spec,
        seq_lens=torch.tensor(lens, dtype=torch.int32),
        cu_q=cu_q,
        pos=torch.from_numpy(pos),
        row_seq=torch.from_numpy(row_seq),
        q_idx=q_idx, q_scale=q_scale,
        k_idx=k_idx, k_scale=k_scale, k_pages=k_pages,
        w=w_t, q=q_t, kv=kv_t, page_table=page_table, n_max=n_max)


def small_spec(base: Spec, **kw) -> Spec:
    """A reduced copy of `base` for parity runs the oracle finishes in seconds."""
    return base.replace(**kw)
