#!/usr/bin/env python
"""Throughput of the DSA hot path (lightning indexer -> top-k -> sparse MQA
attention) on the 128K-context paged decode workload: B = 16 sequences of
96K-128K keys, page size 64, k = 2048, 64 FP8 indexer heads of 128 dims,
128 bf16 query heads over 576-wide latent rows.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of all three stages over the batch (each sequence's newest
token). Prints one JSON line (rank 0). Under torchrun each rank processes its
own batch (weak scaling, no data-path collective); the step time is the max over
ranks. --impl reference times the CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "DSA tokens/s (indexer+top-k+sparse attn) at 128K decode, % of roofline"
UNIT = "tokens/s"
WORKLOAD = "paged_decode_b16_ctx96k_128k"


def captured_traffic(name="indexer_fp8_traffic.txt"):
    """DRAM bytes per launch from a committed ncu capture, or None once the
    kernel's sources differ from the ones that capture measured."""
    path = os.path.join(ROOT, "profiles", name)
    try:
        kv = dict(line.split("=", 1) for line in open(path).read().splitlines()
                  if line and not line.startswith("#") and "=" in line)
        h = hashlib.sha256()
        for f in kv["sources"].split():
            with open(os.path.join(ROOT, f), "rb") as fh:
                h.update(fh.read())
        return int(kv["traffic_bytes_per_launch"]) if h.hexdigest() == kv["sha256"].strip() else None
    except (OSError, KeyError, ValueError):
        return None


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler(threading.Thread):
    """Samples SM clock and clock-event reasons through NVML (read-only)."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period=0.005):
        super().__init__(daemon=True)
        self.samples = []
        self.period = period
        self.stop_flag = threading.Event()
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml as N
            N.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            self.h = N.nvmlDeviceGetHandleByPciBusId(bus)
            self.N = N
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(self.h, N.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = repr(e)

    def run(self):
        if not self.ok:
            return
        N = self.N
        while not self.stop_flag.is_set():
            try:
                sm = N.nvmlDeviceGetClockInfo(self.h, N.NVML_CLOCK_SM)
                rs = N.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), sm, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def summary(self, t0=None, t1=None):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        s = [x for x in self.samples if (t0 is None or x[0] >= t0) and (t1 is None or x[0] <= t1)]
        if not s:
            s = self.samples
        loaded = [x for x in s if not (x[2] & 0x1)] or s
        mhz = statistics.median([x[1] for x in loaded]) if loaded else None
        bits = 0
        for x in loaded:
            bits |= x[2]
        reasons = [n for b, n in self.REASONS.items() if bits & b and b != 0x1]
        return {"sm_mhz": mhz, "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(loaded)}


# ------------------------------------------------------------------ work accounting
def algorithmic_bytes(inp, fused=True):
    """Bytes each stage must move (inputs read once, outputs written once). The
    fused indexer writes no score rows; "topk" keeps the unfused definition (each
    score read once, each index written once), the one the top-k + attention
    target is stated in."""
    s = inp.spec
    lens = [int(x) for x in inp.seq_lens.tolist()]
    B, tot = len(lens), sum(lens)
    sel = sum(min(s.k, L) for L in lens)
    pages = sum((L + s.page_size - 1) // s.page_size for L in lens) if s.page_size else 0
    idx_bytes = (tot * (s.d_I + 4)            # FP8 key rows + per-key scale
                 + B * (s.H_I * s.d_I + 4 + s.H_I * 4)   # query heads, scale, weights
                 + pages * 4                  # page-table entries
                 + (0 if fused else tot * 4))  # scores written (unfused only)
    topk_bytes = tot * 4 + B * s.k * 4
    attn_bytes = (sel * s.Dk * 2              # gathered latent rows
                  + B * s.H * s.Dk * 2        # queries
                  + B * s.k * 4 + pages * 4   # indices, page table
                  + B * s.H * s.Dv * 2 + B * s.H * 4)  # output, lse
    return {"indexer": idx_bytes, "topk": topk_bytes, "attn": attn_bytes}


# ------------------------------------------------------------------ oracle (CPU) leg
def path_flops(lens, spec):
    """Flops of the whole path for one query row at each context length: the
    indexer over every key, attention over min(k, len) selected rows."""
    return [L * 2 * spec.H_I * spec.d_I + min(spec.k, L) * 2 * spec.H * (spec.Dk + spec.Dv) for L in lens]


def oracle_steps(inp, budget_s):
    """Whole steps (every query row, whole path) of the C++ oracle until `budget_s`
    is spent: (steps, seconds, threads)."""
    from oracle import dsa_oracle as O
    from tests.case_utils import case_from_inputs
    case = case_from_inputs(inp)
    rows = list(range(inp.T))
    n = 0
    t0 = time.perf_counter()
    while True:
        O.forward_rows(case, rows, want_scores=False)
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    return n, time.perf_counter() - t0, O.threads()


# ------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill FP8 indexer measurement")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip timing the other four workloads (stages, dsa_forward, roofline fractions)")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip timing the sparse-attention backward on the step's selection")
    ap.add_argument("--all-configs", action="store_true",
                    help="time every workload (stages, forward, roofline fractions), one JSON line each")
    ap.add_argument("--only", default=None,
                    help="with --all-configs: time this one workload (by name) only")
    ap.add_argument("--len-range", type=int, nargs=2, default=None,
                    help="override the context-length range (profiling on a smaller case)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    from sparse_long_context_04_b200 import dist as X
    world, rank, local = X.rank_info()

    if args.impl == "reference":
        return run_reference(args, world, rank)

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    X.init("nccl", dev)

    from sparse_long_context_04_b200 import build as B
    if rank == 0:
        B.build()
    X.barrier()
    from sparse_long_context_04_b200 import device as G
    from sparse_long_context_04_b200 import dsa as D
    from sparse_long_context_04_b200 import workloads as W

    if args.all_configs:
        if rank == 0:
            for line in all_configs(dev, G, D, W, only=args.only).values():
                print(json.dumps(dict(mode="all_configs", **line)), flush=True)
        X.finish()
        return

    spec = W.WORKLOADS[WORKLOAD]
    spec = spec.replace(seed=X.rank_seed(spec.seed, rank))
    if args.len_range:
        spec = spec.replace(len_range=tuple(args.len_range))
    inp = W.make_inputs(spec)
    dc = G.to_device(inp, dev)
    T, s = dc.T, spec
    scores = torch.empty((T, dc.ld), dtype=torch.float32, device=dev)
    idx = torch.empty((T, s.k), dtype=torch.int32, device=dev)
    out = torch.empty((T, s.H, s.Dv), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((T, s.H), dtype=torch.float32, device=dev)
    wsn = D.dsa_sparse_mqa_attn_workspace_size(T, s.H, s.Dv, s.k, dc.q)
    ws = torch.empty(max(wsn, 256), dtype=torch.uint8, device=dev)
    # the fused indexer -> top-k (dsa_indexer_candidates + dsa_topk_from_candidates),
    # timed beside the step for comparison: candidates and their histogram instead
    # of score rows
    hist = torch.empty((T, 4096), dtype=torch.int32, device=dev)
    cand_s = torch.empty((T, dc.ld), dtype=torch.float32, device=dev)
    cand_p = torch.empty((T, dc.ld), dtype=torch.int32, device=dev)
    cand_n = torch.empty((T,), dtype=torch.int32, device=dev)
    # indexer, top-k, then attention: a kernel and a split-merge kernel per chunk of 74 rows
    launches_per_step = 2 + 2 * ((T + 73) // 74)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        D.dsa_indexer_scores(dc.q_idx, dc.q_scale, dc.k_idx, dc.k_scale, dc.w, dc.layout, scores)
        if ev is not None:
            ev[1].record(stream)
        D.dsa_topk(scores, s.k, dc.layout, idx)
        if ev is not None:
            ev[2].record(stream)
        D.dsa_sparse_mqa_attn(dc.q, dc.kv, idx, dc.layout, out, lse, s.softmax_scale, ws)
        if ev is not None:
            ev[3].record(stream)

    def fused_step():
        D.dsa_indexer_candidates(dc.q_idx, dc.q_scale, dc.k_idx, dc.k_scale, dc.w, dc.layout, s.k, hist, cand_s,
                                 cand_p, cand_n)
        D.dsa_topk_from_candidates(cand_s, cand_p, cand_n, hist, s.k, dc.layout, idx)
        D.dsa_sparse_mqa_attn(dc.q, dc.kv, idx, dc.layout, out, lse, s.softmax_scale, ws)

    def fused_steps(n=200):
        """Whole steps on the fused pair, back to back like the timed ones (ms per step)."""
        for _ in range(5):
            fused_step()
        torch.cuda.synchronize(dev)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(n):
            fused_step()
        f1.record(stream)
        torch.cuda.synchronize(dev)
        return f0.elapsed_time(f1) / n

    def fused_stages(reps=40):
        """The fused pair's two stages, CUDA events around each."""
        evs_f = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
        for e3 in evs_f:
            e3[0].record(stream)
            D.dsa_indexer_candidates(dc.q_idx, dc.q_scale, dc.k_idx, dc.k_scale, dc.w, dc.layout, s.k, hist, cand_s,
                                     cand_p, cand_n)
            e3[1].record(stream)
            D.dsa_topk_from_candidates(cand_s, cand_p, cand_n, hist, s.k, dc.layout, idx)
            e3[2].record(stream)
        torch.cuda.synchronize(dev)
        return {"indexer": sum(e3[0].elapsed_time(e3[1]) for e3 in evs_f) / reps * 1e3,
                "topk": sum(e3[1].elapsed_time(e3[2]) for e3 in evs_f) / reps * 1e3}

    sampler = ClockSampler(local)
    sampler.start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if D.dsa_get_device_error() != D.DSA_OK:
        raise RuntimeError("device error during warm-up")

    # Stage events on every 8th step only: an event between two kernels ends the
    # overlap of one kernel's tail with the next one's launch (programmatic
    # dependent launch), so the other steps run back to back as a user's would.
    every = 8
    probed = list(range(0, args.steps, every))
    evs = {i: [torch.cuda.Event(enable_timing=True) for _ in range(4)] for i in probed}
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    X.barrier()
    torch.cuda.synchronize(dev)
    wt0 = time.perf_counter()
    start.record(stream)
    for i in range(args.steps):
        step(evs.get(i))
    end.record(stream)
    torch.cuda.synchronize(dev)
    wt1 = time.perf_counter()
    X.barrier()
    ms = start.elapsed_time(end)
    stage_ms = [sum(evs[i][j].elapsed_time(evs[i][j + 1]) for i in probed) / len(probed) for j in range(3)]
    ms = X.max_over_ranks(ms, dev)
    if D.dsa_get_device_error() != D.DSA_OK:
        raise RuntimeError("device error during timing")
    fused = fused_stages()
    kept = int(cand_n.sum())
    fused_ms = fused_steps()
    step()                       # the score rows and selection the indexer loss below reads
    torch.cuda.synchronize(dev)
    if D.dsa_get_device_error() != D.DSA_OK:
        raise RuntimeError("device error in the fused stages")

    # ---- end to end through dsa_forward with host buffers. Two slots of per-step
    # device inputs and outputs: step i+1's inputs cross PCIe (own stream) while
    # step i computes, and step i's output returns (another stream) while step
    # i+1 computes. Every step still copies its inputs in and its result out. The
    # step's inputs sit in one pinned buffer (one copy per step, each tensor at a
    # 256-byte offset), and so do its output and log-sum-exp.
    srcs = {n: getattr(dc, n) for n in ("q_idx", "q_scale", "w", "q") if getattr(dc, n) is not None}
    srcs["seq_lens"] = dc.layout.seq_lens
    if dc.layout.page_table is not None:
        srcs["page_table"] = dc.layout.page_table

    def pack_layout(shapes):
        offs, off = {}, 0
        for n, (shape, dtype) in shapes.items():
            nb = math.prod(shape) * torch.empty((), dtype=dtype).element_size()
            offs[n] = (off, nb, shape, dtype)
            off = (off + nb + 255) // 256 * 256
        return offs, off

    def views(buf, offs):
        return {n: buf[o:o + nb].view(dt).view(shape) for n, (o, nb, shape, dt) in offs.items()}

    in_offs, in_bytes = pack_layout({n: (tuple(t.shape), t.dtype) for n, t in srcs.items()})
    out_offs, out_bytes = pack_layout({"out": ((T, s.H, s.Dv), torch.bfloat16), "lse": ((T, s.H), torch.float32)})
    host_in = torch.zeros(in_bytes, dtype=torch.uint8).pin_memory()
    for n, v in views(host_in, in_offs).items():
        v.copy_(srcs[n].cpu())
    dev_in = [torch.empty(in_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    dev_out = [torch.empty(out_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    host_out = [torch.empty(out_bytes, dtype=torch.uint8).pin_memory() for _ in range(2)]

    def slot_forward(j):
        v, o = views(dev_in[j], in_offs), views(dev_out[j], out_offs)
        lay = dc.layout
        nl = D.Layout(v["seq_lens"], lay.c.n_max, None, v.get("page_table"), lay.c.page_size, lay.c.num_pages)
        c = dataclasses.replace(dc, q_idx=v["q_idx"], q_scale=v.get("q_scale"), w=v["w"], q=v["q"], layout=nl)
        return G.Forward(c, keep_idx=False, out=o["out"], lse=o["lse"])

    fws = [slot_forward(0), slot_forward(1)]
    h2d, d2h = in_bytes, out_bytes
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready, in_free = [ev(), ev()], [ev(), ev()]
    out_ready, out_free = [ev(), ev()], [ev(), ev()]
    for e in in_free + out_free:
        e.record(stream)

    def e2e_step(i):
        j = i & 1
        with torch.cuda.stream(s_in):            # inputs of step i into slot j
            s_in.wait_event(in_free[j])
            dev_in[j].copy_(host_in, non_blocking=True)
            in_ready[j].record(s_in)
        stream.wait_event(in_ready[j])          # compute step i
        stream.wait_event(out_free[j])
        fws[j](stream)
        in_free[j].record(stream)
        out_ready[j].record(stream)
        with torch.cuda.stream(s_out):           # result of step i back to the host
            s_out.wait_event(out_ready[j])
            host_out[j].copy_(dev_out[j], non_blocking=True)
            out_free[j].record(s_out)

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    X.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    for i in range(args.e2e_steps):
        e2e_step(i)
    s_out_done = torch.cuda.Event()
    s_out_done.record(s_out)
    stream.wait_event(s_out_done)               # the last result is on the host inside the timed region
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = X.max_over_ranks(e0.elapsed_time(e1), dev)
    # the last step's result on the host equals the stage-by-stage path's output
    # for the same inputs (the same kernels run in both)
    got = views(host_out[(args.e2e_steps - 1) & 1], out_offs)["out"]
    if not torch.equal(got.view(torch.int16), out.cpu().view(torch.int16)):
        raise RuntimeError("dsa_forward's result copied to the host differs from the staged path's")
    # ---- indexer loss on the last step's selection (a training-side call, outside
    # the metric's step): KL(heads' mean attention || softmax of the selected scores).
    # Its 40 MB of inputs fit in L2, so L2 is flushed before every timed call.
    kl_loss = torch.empty(T, dtype=torch.float32, device=dev)
    kl_grad = torch.empty((T, s.k), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        D.dsa_indexer_kl(dc.q, dc.kv, idx, dc.layout, lse, scores, kl_loss, s.softmax_scale, kl_grad)
    torch.cuda.synchronize(dev)
    kl_reps = 20
    kl_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(kl_reps)]
    for r in range(kl_reps):
        flush.fill_(r & 0xFF)
        kl_ev[r][0].record(stream)
        D.dsa_indexer_kl(dc.q, dc.kv, idx, dc.layout, lse, scores, kl_loss, s.softmax_scale, kl_grad)
        kl_ev[r][1].record(stream)
    torch.cuda.synchronize(dev)
    kl_us = sum(a.elapsed_time(b) for a, b in kl_ev) / kl_reps * 1e3
    kl_valid = int((idx >= 0).sum())
    del flush
    if D.dsa_get_device_error() != D.DSA_OK:
        raise RuntimeError("device error during the indexer loss")
    # ---- sparse-attention backward on the last step's selection and output (a
    # training-side call, outside the metric's step), L2 flushed before each call
    bwd = None
    if not args.no_backward:
        g = torch.Generator(device=dev).manual_seed(4321)
        dout = torch.randn((T, s.H, s.Dv), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
        dq = torch.zeros((T, s.H, s.Dk), dtype=torch.float32, device=dev)
        dkv = torch.zeros(tuple(dc.kv.shape), dtype=torch.float32, device=dev)
        bws = torch.empty(D.dsa_sparse_mqa_attn_backward_workspace_size(T), dtype=torch.uint8, device=dev)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        for _ in range(args.warmup):
            D.dsa_sparse_mqa_attn_backward(dc.q, dc.kv, idx, dc.layout, out, dout, lse, dq, dkv, s.softmax_scale, bws)
        torch.cuda.synchronize(dev)
        b_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(10)]
        for r, (e0b, e1b) in enumerate(b_ev):
            flush.fill_(r & 0xFF)
            e0b.record(stream)
            D.dsa_sparse_mqa_attn_backward(dc.q, dc.kv, idx, dc.layout, out, dout, lse, dq, dkv, s.softmax_scale, bws)
            e1b.record(stream)
        torch.cuda.synchronize(dev)
        bwd_us = sum(a.elapsed_time(b) for a, b in b_ev) / len(b_ev) * 1e3
        bwd = (bwd_us, int((idx >= 0).sum()))
        del flush, dkv
        if D.dsa_get_device_error() != D.DSA_OK:
            raise RuntimeError("device error during the attention backward")
    # ---- cache write of the step's new tokens (the other half of a decode loop):
    # each sequence's newest indexer key quantised into its page, its latent row copied
    g = torch.Generator(device=dev).manual_seed(1234)
    k_new = torch.randn((T, s.d_I), generator=g, device=dev, dtype=torch.float32)
    kv_new = torch.randn((T, s.Dk), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    k_scale = None if s.page_size else dc.k_scale
    for _ in range(args.warmup):
        D.dsa_cache_append(k_new, kv_new, dc.layout, dc.k_idx, dc.kv, k_scale)
    torch.cuda.synchronize(dev)
    # one call is a few microseconds of GPU work, less than the host needs to make a
    # call, so the calls are captured in a CUDA graph and the graph is replayed
    per_graph = 20
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(per_graph):
            D.dsa_cache_append(k_new, kv_new, dc.layout, dc.k_idx, dc.kv, k_scale)
    graph.replay()
    torch.cuda.synchronize(dev)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    replays = 10
    a0.record(stream)
    for _ in range(replays):
        graph.replay()
    a1.record(stream)
    torch.cuda.synchronize(dev)
    append_us = a0.elapsed_time(a1) / (replays * per_graph) * 1e3
    del graph
    if D.dsa_get_device_error() != D.DSA_OK:
        raise RuntimeError("device error during the cache write")
    # ---- prefill FP8 indexer (tensor-bound): the 8K-token causal prefill, against
    # the dense FP8 peak measured here
    fp8_tf = measure_fp8_peak(dev) if not args.no_prefill else None
    pf = prefill_indexer(args, dev, G, D, W, fp8_measured=fp8_tf) if not args.no_prefill else None
    # ---- every other workload through the library: stages, dsa_forward, roofline fractions
    cfgs = None
    if not args.no_configs and rank == 0:
        del dc, scores, hist, cand_s, cand_p, cand_n, ws
        torch.cuda.empty_cache()
        cfgs = all_configs(dev, G, D, W, fp8_measured=fp8_tf,
                           names=[n for n in CONFIG_REPS if n != WORKLOAD])
    sampler.stop_flag.set()
    sampler.join()
    if D.dsa_get_device_error() != D.DSA_OK:
        raise RuntimeError("device error during the end-to-end loop")

    X.finish()
    if rank != 0:
        return

    hbm, hbm_src = peaks()
    ab = algorithmic_bytes(inp, fused=False)
    step_s = ms / 1e3 / args.steps
    idx_s = stage_ms[0] / 1e3
    idx_gbs = ab["indexer"] / idx_s / 1e9
    ta_s = (stage_ms[1] + stage_ms[2]) / 1e3
    ta_gbs = (ab["topk"] + ab["attn"]) / ta_s / 1e9
    step_gbs = sum(ab.values()) / step_s / 1e9
    res = {
        "metric": METRIC,
        "value": X.job_rate(world, T, args.steps, ms),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3 indexer + bf16 attention (fp32 accumulate)",
        "data": "synthetic (seeded; shapes and planted structure of the 128K paged decode workload)",
        "config": {
            "workload": WORKLOAD if not args.len_range else WORKLOAD + "@len%d-%d" % tuple(args.len_range),
            "batch_per_gpu": T, "context": "uniform %d..%d" % spec.len_range,
            "keys_total_per_gpu": int(inp.seq_lens.sum()), "page_size": s.page_size, "k": s.k,
            "H_I": s.H_I, "d_I": s.d_I, "H": s.H, "Dk": s.Dk, "Dv": s.Dv,
            "parallelism": f"dp{world} (independent sequences per rank)",
            "l2": "inputs larger than L2: the 242 MB paged indexer-key cache is streamed every step",
        },
        "stages_us": {"indexer": stage_ms[0] * 1e3, "topk": stage_ms[1] * 1e3, "attention": stage_ms[2] * 1e3,
                      "probed_steps": len(probed),
                      "path": "score rows (dsa_indexer_scores) + cluster top-k (dsa_topk), as dsa_forward's default"},
        "fused_topk": {"ms_per_step": fused_ms, "tokens_per_s": T / (fused_ms / 1e3),
                       "stages_us": fused, "candidates_kept": kept, "keys": int(inp.seq_lens.sum()),
                       "kept_frac": kept / int(inp.seq_lens.sum()),
                       "note": "dsa_indexer_candidates + dsa_topk_from_candidates (no score rows) + attention: "
                               "200 whole steps back to back; stage times from 40 more with events around each "
                               "stage; same selection as the step's"},
        "roofline": {
            "bound": "hbm", "kernel": "indexer_fp8_kernel (decode, N=64)",
            "achieved": idx_gbs, "peak": hbm, "unit": "GB/s", "frac": idx_gbs / hbm,
            "peak_source": f"{hbm_src} (MEASURED_PEAKS.json hbm_gbs)" if hbm_src == "measured" else "fallback 6.65 TB/s",
            "algorithmic_bytes_per_launch": ab["indexer"],
            "traffic": captured_traffic(),
        },
        "topk_attn_roofline": {"achieved": ta_gbs, "frac": ta_gbs / hbm,
                               "algorithmic_bytes": ab["topk"] + ab["attn"]},
        "step_roofline": {"achieved": step_gbs, "frac": step_gbs / hbm, "algorithmic_bytes": sum(ab.values())},
        "fp8_indexer_prefill": pf,
        "configs": cfgs,
        "fp8_peak_tflops": {"measured": fp8_tf, "datasheet": FP8_DATASHEET_TFLOPS,
                            "how": "torch._scaled_mm e4m3 x e4m3 -> bf16, 8192^3, best of 10, CUDA events"},
        "e2e": {"value": X.job_rate(world, T, args.e2e_steps, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
                "api": "dsa_forward",
                "pipeline": "two slots: step i+1's inputs in and step i's result out on their own "
                            "streams while step i computes; every step copies both"},
        "cache_append": {"us": append_us, "rows": T, "api": "dsa_cache_append",
                         "bytes": T * (s.d_I * 4 + s.d_I + 4 + 4 * s.Dk),
                         "note": "per call, 20 calls per CUDA graph replay; not part of the metric's step"},
        "indexer_kl": indexer_kl_summary(kl_us, T, s, kl_valid, hbm, hbm_src),
        **({"attn_backward": attn_backward_summary(bwd[0], T, s, bwd[1], hbm, hbm_src)} if bwd else {}),
        "gpu_launches": launches_per_step * args.steps,
        "clocks": sampler.summary(wt0, wt1),
    }
    if world == 1 and not args.no_cpu_baseline:
        steps_c, secs, cores = oracle_steps(inp, args.cpu_budget)
        res["cpu_baseline"] = {
            "value": steps_c * T / secs, "unit": UNIT, "cores": cores, "kind": "oracle (C++, fp64)",
            "sample": f"{steps_c} whole steps of this workload ({T} query rows each, indexer + top-k + attention), "
                      f"rows spread over {cores} threads, {secs:.1f} s"}
    print(json.dumps(res), flush=True)


def indexer_kl_summary(us, T, s, valid, hbm, hbm_src):
    """Per-call time of the indexer loss and its HBM roofline: each call reads the
    selected latent rows, the query rows, the selection, the per-head log-sum-exp
    and the selected scores, and writes the gradient and the loss."""
    algo = (valid * (s.Dk * 2 + 4) + T * (s.H * s.Dk * 2 + s.H * 4 + 4)
            + 2 * T * s.k * 4)
    gbs = algo / (us * 1e-6) / 1e9
    return {"us": us, "rows": T, "k": s.k, "api": "dsa_indexer_kl", "kernel": "indexer_kl_kernel",
            "bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
            "peak_source": f"{hbm_src} (MEASURED_PEAKS.json hbm_gbs)" if hbm_src == "measured"
            else "fallback 6.65 TB/s",
            "algorithmic_bytes_per_call": algo, "flops": 2.0 * valid * s.H * s.Dk,
            "traffic": captured_traffic("indexer_kl_traffic.txt"),
            "note": "per call (loss and gradient), L2 flushed before each of 20 timed calls; "
                    "not part of the metric's step"}


def attn_backward_summary(us, T, s, valid, hbm, hbm_src):
    """Per-call time of the sparse-attention backward against HBM bandwidth: each
    call reads every selected latent row, the query, output-gradient and output
    blocks, and adds into dq and into the selected rows of dkv (fp32, read and
    written)."""
    algo = (valid * (s.Dk * 2 + 2 * s.Dk * 4)          # row gathered, its dkv row read and written
            + T * s.H * (s.Dk * 2 + 2 * s.Dv * 2 + 4)   # q, dO, o, lse
            + T * s.H * s.Dk * 4 * 2                     # dq read and written
            + T * s.k * 4)                               # the selection
    gbs = algo / (us * 1e-6) / 1e9
    flops = 2.0 * valid * s.H * (3 * s.Dk + 2 * s.Dv)     # S, dP, dKV (two terms), dQ
    return {"us": us, "rows": T, "k": s.k, "api": "dsa_sparse_mqa_attn_backward", "kernel": "attn_bwd_kernel",
            "bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
            "peak_source": f"{hbm_src} (MEASURED_PEAKS.json hbm_gbs)" if hbm_src == "measured"
            else "fallback 6.65 TB/s",
            "algorithmic_bytes_per_call": algo, "flops": flops,
            "note": "per call (delta kernel included), L2 flushed before each of 10 timed calls; "
                    "not part of the metric's step"}


FP8_DATASHEET_TFLOPS = 4500.0   # dense e4m3, per GPU (context only)


def measure_fp8_peak(dev, n=8192, reps=10):
    """Dense e4m3 x e4m3 -> bf16 GEMM throughput of torch._scaled_mm at n^3
    (2 n^3 flop), best of `reps` CUDA-event-timed calls after warm-up: the same
    method as the measured bf16 peak, for the FP8 roofline. None if the call is
    unavailable."""
    try:
        g = torch.Generator(device=dev).manual_seed(7)
        a = torch.randn((n, n), generator=g, device=dev).to(torch.float8_e4m3fn)
        b = torch.randn((n, n), generator=g, device=dev).to(torch.float8_e4m3fn).t()
        one = torch.ones((), dtype=torch.float32, device=dev)
        for _ in range(3):
            torch._scaled_mm(a, b, one, one, out_dtype=torch.bfloat16)
        torch.cuda.synchronize(dev)
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._scaled_mm(a, b, one, one, out_dtype=torch.bfloat16)
            e1.record()
            torch.cuda.synchronize(dev)
            best = min(best, e0.elapsed_time(e1))
        del a, b
        return 2.0 * n ** 3 / (best / 1e3) / 1e12
    except Exception:
        return None


def fp8_peak(measured):
    """(peak TFLOP/s, where it comes from) for the FP8 roofline."""
    if measured:
        return measured, "measured in this run: torch._scaled_mm e4m3 8192^3, best of 10"
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return 2 * float(json.load(f)["bf16_tflops"]), "estimate: 2x measured bf16 burst (nominal ratio)"
    except Exception:
        return 2 * 1590.0, "estimate: 2x fallback bf16"


def prefill_indexer(args, dev, G, D, W, reps=20, fp8_measured=None):
    """Event-timed FP8 indexer over the causal 8192-token prefill: 16384 flop per
    (query, earlier key) pair, against the dense FP8 peak measured in the same run
    (and, for context, the 4.5 PFLOP/s datasheet figure)."""
    spec = W.PREFILL_8K
    inp = W.make_inputs(spec)
    dc = G.to_device(inp, dev)
    scores = torch.empty((dc.T, dc.ld), dtype=torch.float32, device=dev)
    for _ in range(3):
        G.indexer(dc, scores)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        G.indexer(dc, scores)
    e1.record()
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / reps
    L = int(inp.seq_lens[0])
    pairs = L * (L + 1) // 2
    flops = pairs * 2 * spec.H_I * spec.d_I
    tf = flops / (ms / 1e3) / 1e12
    peak, src = fp8_peak(fp8_measured)
    return {"workload": spec.name, "us": ms * 1e3, "pairs": pairs, "tflops": tf, "peak_tflops": peak,
            "frac": tf / peak, "peak_source": src, "frac_of_datasheet": tf / FP8_DATASHEET_TFLOPS,
            "datasheet_tflops": FP8_DATASHEET_TFLOPS, "kernel": "indexer_fp8_kernel (prefill, N=256)"}


def config_line(spec, reps, dev, G, D, W, hbm, bf16, fp8):
    """One workload through the library: per-stage CUDA-event times (each stage
    called on its own over every row, L2 warm), the composed dsa_forward, tokens/s
    and each stage against its roofline (the larger of algorithmic bytes / measured
    HBM bandwidth and flops / the dtype's measured dense peak)."""
    inp = W.make_inputs(spec, big_q_device=dev)
    dc = G.to_device(inp, dev)
    T, s = dc.T, spec
    pos = inp.pos.to(torch.int64)
    n_pairs = int((pos + 1).sum())
    n_sel = int(torch.clamp(pos + 1, max=s.k).sum())
    lens = [int(x) for x in inp.seq_lens.tolist()]
    scores = torch.empty((T, dc.ld), dtype=torch.float32, device=dev)
    idx = torch.empty((T, s.k), dtype=torch.int32, device=dev)
    out = torch.empty((T, s.H, s.Dv), dtype=dc.q.dtype, device=dev)
    lse = torch.empty((T, s.H), dtype=torch.float32, device=dev)
    wsn = D.dsa_sparse_mqa_attn_workspace_size(T, s.H, s.Dv, s.k, dc.q)
    ws = torch.empty(max(wsn, 256), dtype=torch.uint8, device=dev)
    stages = {
        "indexer": lambda: D.dsa_indexer_scores(dc.q_idx, dc.q_scale, dc.k_idx, dc.k_scale, dc.w, dc.layout, scores),
        "topk": lambda: D.dsa_topk(scores, s.k, dc.layout, idx),
        "attention": lambda: D.dsa_sparse_mqa_attn(dc.q, dc.kv, idx, dc.layout, out, lse, s.softmax_scale, ws),
    }
    ms = {}
    for name, fn in stages.items():
        for _ in range(2):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize(dev)
        ms[name] = e0.elapsed_time(e1) / reps
    del scores
    fw = G.Forward(dc, keep_idx=False)
    for _ in range(2):
        fw()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fw()
    e1.record()
    torch.cuda.synchronize(dev)
    fwd_ms = e0.elapsed_time(e1) / reps
    if D.dsa_get_device_error() != D.DSA_OK:
        raise RuntimeError(f"device error on {spec.name}")
    line = {"workload": spec.name, "query_rows": T, "tokens_per_s": T / (fwd_ms / 1e3), "forward_ms": fwd_ms,
            "stages_ms": ms, "dtype": "fp32" if not s.fp8 else "e4m3 indexer + bf16 attention"}
    if s.fp8:
        kbytes = sum(lens) * (s.d_I + 4) + T * (s.H_I * s.d_I + 4 + 4 * s.H_I)
        roof = {
            "indexer": max((kbytes + n_pairs * 4) / hbm / 1e6, 2 * s.H_I * s.d_I * n_pairs / fp8 / 1e9),
            "topk": (n_pairs * 4 + T * s.k * 4) / hbm / 1e6,
            "attention": max((n_sel * s.Dk * 2 + T * s.H * (s.Dk + s.Dv) * 2 + T * s.H * 4) / hbm / 1e6,
                             2 * s.H * (s.Dk + s.Dv) * n_sel / bf16 / 1e9),
        }
        line["roofline_ms"] = roof
        line["frac"] = {k: roof[k] / ms[k] for k in roof}
        line["forward_frac"] = sum(roof.values()) / fwd_ms
        line["bound"] = "hbm" if s.mode == "decode" else "tensor (fp8 indexer, bf16 attention)"
    del dc, idx, out, lse, ws, fw, inp
    torch.cuda.empty_cache()
    return line


CONFIG_REPS = {"tiny_fp32_prefill_L256": 20, "decode_b32_ctx32k": 50, "prefill_L8192": 5,
               "prefill_2x32768_ar1": 2, "paged_decode_b16_ctx96k_128k": 50}


def all_configs(dev, G, D, W, only=None, fp8_measured=None, names=None):
    """Every workload once (or `only`): a dict name -> config_line."""
    hbm, _ = peaks()
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            bf16 = float(json.load(f)["bf16_tflops"])
    except Exception:
        bf16 = 1590.0
    fp8, fp8_src = fp8_peak(fp8_measured if fp8_measured else measure_fp8_peak(dev))
    res = {}
    for spec in (W.TINY, W.DECODE_32K, W.PREFILL_8K, W.PREFILL_2X32K, W.PAGED_DECODE_128K):
        if (only and spec.name != only) or (names is not None and spec.name not in names):
            continue
        line = config_line(spec, CONFIG_REPS[spec.name], dev, G, D, W, hbm, bf16, fp8)
        line["peaks"] = {"hbm_gbs": hbm, "bf16_tflops": bf16, "fp8_tflops": fp8, "fp8_source": fp8_src}
        res[spec.name] = line
    return res


def run_reference(args, world, rank):
    """The CPU oracle (C++, fp64) as it stands, on a bounded sample of the same
    workload: each step runs the whole path for every query row of the batch
    (rows spread over the host's threads) over a truncated context, sized so that
    warm-up and timed steps take about two minutes; the rate is scaled to the
    full contexts by the exact flops of the path per row."""
    if rank != 0:
        return
    from oracle import dsa_oracle as O
    from sparse_long_context_04_b200 import workloads as W
    from tests.case_utils import case_from_inputs

    spec = W.WORKLOADS[WORKLOAD]
    inp = W.make_inputs(spec)
    case = case_from_inputs(inp)
    lens = [int(x) for x in inp.seq_lens.tolist()]
    rows = list(range(inp.T))
    t_probe = time.perf_counter()
    O.forward_rows(case, rows, want_scores=False)
    full_s = time.perf_counter() - t_probe
    n_steps = args.steps + args.warmup
    frac = min(1.0, 120.0 / max(1e-9, n_steps * full_s))
    cut = [max(min(spec.k, L), int(L * frac)) for L in lens]   # keys each row scores in a sample step
    sample = dict(case)
    sample["pos"] = np.asarray([c - 1 for c in cut], dtype=np.int32)
    work_ratio = sum(path_flops(cut, spec)) / sum(path_flops(lens, spec))
    for _ in range(args.warmup):
        O.forward_rows(sample, rows, want_scores=False)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.forward_rows(sample, rows, want_scores=False)
    secs = time.perf_counter() - t0
    value = args.steps * inp.T * work_ratio / secs     # rows/s at the full contexts
    cores = O.threads()
    res = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; shapes and planted structure of the 128K paged decode workload)",
        "config": {"workload": WORKLOAD, "batch_per_gpu": inp.T, "k": spec.k, "page_size": spec.page_size},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle (C++, fp64)",
                         "sample": f"per step: all {inp.T} query rows, whole path, each row's context cut to "
                                   f"{frac:.3f} of its length (at least k); scaled to the full contexts by the "
                                   f"path's flops per row (sample/full = {work_ratio:.4f})"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
