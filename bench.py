"""Benchmark of the sparse attention backward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload 4]

One step = one full sfa_grad call (zero-init, index compaction, rowsum(dO*O),
key-row expansion, the fused tensor-core backward, the dQuery and dKey/dValue
casts) over one batch of the workload, inputs resident in HBM.  The metric is
TFLOP/s with the 5-GEMM count (5504 FLOP per valid (query row, head, key)).

N > 1 (torchrun), sparse workloads: the workload's query rows are split into N
contiguous ranges of equal work (valid (row, key) pairs); every rank holds the
whole (identically generated) problem, runs the backward of its rows into a
key-side accumulator (sfa_grad_rows), the ranks sum the accumulators with one
NCCL all-reduce (int64 fixed point in deterministic mode: exact), and each rank
casts it (sfa_dkv_finalize).  One step = that whole sharded backward; value =
the workload's FLOP / the max over ranks of the timed region ("scaling":
"strong").  The dense FA workload (2) runs independent replicas ("weak").

--impl reference times the CPU oracle (the plain numpy definition) on a
bounded sample of the same workload on the host cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-attn backward TFLOP/s (bf16, 5-GEMM count) and % of B200 tensor peak"
FLOP_PER_TRIPLE = 5504
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}


# committed ncu summaries: (summary file, kernel sources whose hash it records)
PROFILE_SUMMARIES = {
    4: ("sfa_bwd_pair_kernel_workload4.md", ("sfa_pair.cu", "tc_common.cuh")),
    3: ("sfa_bwd_fused_kernel_workload3.md", ("sfa_fused.cu", "tc_common.cuh")),
    5: ("sfa_bwd_fused_kernel_workload5.md", ("sfa_fused.cu", "tc_common.cuh")),
    2: ("fa_bwd_fused_kernel_workload2.md", ("fa_fused.cu", "tc_common.cuh")),
    "fwd4": ("sfa_fwd_fused_kernel_workload4.md", ("sfa_fwd_fused.cu", "tc_common.cuh")),
    "lig": ("lig_fused_kernel_indexer.md", ("lig_fused.cu", "tc_common.cuh")),
}


def kernel_source_hash(sources):
    import hashlib
    h = hashlib.sha256()
    for f in sources:
        with open(os.path.join(ROOT, "sparse_attention_backward_sfa_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic(workload):
    """DRAM bytes per launch of the workload's main kernel from the committed ncu
    summary, or None when there is none or the kernel sources changed since the capture."""
    if workload not in PROFILE_SUMMARIES:
        return None
    name, sources = PROFILE_SUMMARIES[workload]
    try:
        txt = open(os.path.join(ROOT, "profiles", name)).read()
    except OSError:
        return None
    vals = dict(re.findall(r"^(traffic_bytes_per_launch|kernel_source_sha256):\s*(\S+)", txt, re.M))
    if vals.get("kernel_source_sha256") != kernel_source_hash(sources):
        return None
    try:
        return float(vals["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """Samples nvidia-smi clocks / throttle reasons in the background."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.rows = []
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                                      "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=5)
                if out.returncode == 0 and out.stdout.strip():
                    self.rows.append([x.strip() for x in out.stdout.strip().split(",")])
            except Exception:
                pass
            self._stop.wait(0.2)

    def __enter__(self):
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join(timeout=6)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in self.rows:
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(self.rows)}


# ---------------------------------------------------------------------------
SEQS = None  # optional smaller case of workload 4 or 5 (--seqs, for profiling captures)


def build_problem(workload: int, seed_offset: int, device):
    from workloads import make_device_problem
    p = make_device_problem(workload, device=device,
                            seed=None if seed_offset == 0 else 2000 + workload + 7919 * seed_offset,
                            seqs=SEQS if workload in (4, 5) else None)
    return p


def kw(p):
    return dict(scale=p.scale, sparse_block_size=p.block_size, layout=p.layout, sparse_mode=p.sparse_mode,
                actual_seq_lengths_q=p.seqlens_q, actual_seq_lengths_kv=p.seqlens_kv)


def paired_work_fraction(p, S):
    """Share of the valid (row, key) pairs in rows the paired kernel takes: rows (2m, 2m + 1) of
    one sequence whose block lists (sorted where the library sorts them) are identical and
    non-empty (the library's pairing rule); the rest run on the single-row kernel."""
    import numpy as np
    import torch
    # the library sorts block-sparse lists of topk <= 4096 before pairing; others pair as compacted
    sort = p.block_size > 1 and p.topk <= 4096
    blocks, nb, _, cnt = S.key_rows(p.indices, p.k, p.q, p.q_rope, sparse_block_size=p.block_size,
                                    layout=p.layout, sparse_mode=p.sparse_mode, sorted_blocks=sort,
                                    actual_seq_lengths_q=p.seqlens_q, actual_seq_lengths_kv=p.seqlens_kv)
    T1 = nb.numel()
    M = T1 // 2
    if M == 0:
        return 0.0
    rows = torch.arange(T1, device=nb.device)
    if p.layout == "TND":
        ends = torch.as_tensor(np.asarray(p.seqlens_q if not torch.is_tensor(p.seqlens_q)
                                          else p.seqlens_q.cpu()), dtype=torch.int64, device=nb.device)
        seq = torch.bucketize(rows, ends, right=True)
    else:
        seq = rows // p.S1
    a, b = slice(0, 2 * M, 2), slice(1, 2 * M, 2)
    col = torch.arange(blocks.shape[1], device=nb.device)
    live = col[None, :] < nb[a][:, None]
    same_list = ((blocks[a] == blocks[b]) | ~live).all(dim=1)
    paired = same_list & (nb[a] == nb[b]) & (nb[a] > 0) & (seq[a] == seq[b])
    work = cnt.to(torch.int64)
    tot = int(work.sum())
    return float((work[a] + work[b])[paired].sum()) / tot if tot else 0.0


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import sparse_attention_backward_sfa_b200 as S
    from sparse_attention_backward_sfa_b200 import _native as N

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    lib = N.load()
    sharded = world > 1
    # sharded: every rank builds the same problem and takes its share of the rows
    p = build_problem(args.workload, 0 if sharded else rank, dev)
    out, smax, ssum = S.sfa_fwd(p.q, p.k, p.k, p.indices, p.q_rope, p.k_rope, **kw(p))
    _, _, nr = S.compact_indices(p.indices, p.k, p.q, p.q_rope, sparse_block_size=p.block_size, layout=p.layout,
                                 sparse_mode=p.sparse_mode, actual_seq_lengths_q=p.seqlens_q,
                                 actual_seq_lengths_kv=p.seqlens_kv)
    nr = nr.to(torch.int64).cpu().numpy()
    # the paired kernel serves N1 = 128 (value == key); measured once, outside the timed region
    paired = paired_work_fraction(p, S) if p.N1 == 128 else 0.0
    triples = int(nr.sum()) * p.N1
    flop = triples * FLOP_PER_TRIPLE
    T1 = nr.size
    ranges = S.balanced_row_ranges(nr, world) if sharded else [(0, T1)]
    rb, re_ = ranges[rank]
    flop_rank = int(nr[rb:re_].sum()) * p.N1 * FLOP_PER_TRIPLE
    shape = S.sfa_shape(p.q, p.k, p.q_rope, p.indices, p.layout, p.seqlens_q)
    ws_bytes = S.sfa_grad_workspace_size(shape, p.block_size, p.sparse_mode, p.deterministic)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    outs = (torch.empty_like(p.q), torch.empty_like(p.k), torch.empty_like(p.k), torch.empty_like(p.q_rope),
            torch.empty_like(p.k_rope))
    acc = S.sfa_dkv_accumulator(p.q, p.k, p.q_rope, p.indices, layout=p.layout, deterministic=p.deterministic,
                                actual_seq_lengths_q=p.seqlens_q) if sharded else None
    stream = torch.cuda.current_stream(dev)

    def grad(q, k, idx, do, o, mx, sm, qr, kr, sq, skv):
        if not sharded:
            S.sfa_grad(q, k, k, idx, do, o, mx, sm, qr, kr, deterministic=p.deterministic, workspace=ws, outputs=outs,
                       scale=p.scale, sparse_block_size=p.block_size, layout=p.layout, sparse_mode=p.sparse_mode,
                       actual_seq_lengths_q=sq, actual_seq_lengths_kv=skv)
            return
        dq, dk, dv, dqr, dkr = outs
        acc.zero_()
        dmax = None
        if p.deterministic:  # the fixed-point grid: max|dOut| over every rank's rows
            dmax = S.dout_absmax(do, q, k, qr, idx, layout=p.layout, row_begin=rb, row_end=re_,
                                 actual_seq_lengths_q=sq)
            dist.all_reduce(dmax, op=dist.ReduceOp.MAX)
        S.sfa_grad_rows(q, k, k, idx, do, o, mx, sm, qr, kr, row_begin=rb, row_end=re_, dkv_accum=acc,
                        deterministic=p.deterministic, dout_absmax=dmax, workspace=ws, d_query=dq,
                        d_query_rope=dqr, scale=p.scale, sparse_block_size=p.block_size, layout=p.layout,
                        sparse_mode=p.sparse_mode, actual_seq_lengths_q=sq, actual_seq_lengths_kv=skv)
        dist.all_reduce(acc, op=dist.ReduceOp.SUM)
        S.sfa_dkv_finalize(acc, q, k, qr, idx, layout=p.layout, deterministic=p.deterministic, dout_absmax=dmax,
                           scale=p.scale, actual_seq_lengths_q=sq, outputs=(dk, dv, dkr))

    def step(ev=None):
        if ev is not None:
            N.check(lib.sfa_set_kernel_events(ctypes_ptr(ev[0]), ctypes_ptr(ev[1])))
        grad(p.q, p.k, p.indices, p.dout, out, smax, ssum, p.q_rope, p.k_rope, p.seqlens_q, p.seqlens_kv)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in evs:  # torch creates the CUDA event on first record; the hook needs real handles
        a.record(stream)
        b.record(stream)
    # one event at every step boundary: per-step durations for the median, no extra synchronization
    bnd = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    with ClockSampler(dev.index if "CUDA_VISIBLE_DEVICES" not in os.environ else local_rank) as clk:
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        bnd[0].record(stream)
        for i in range(args.steps):
            step(evs[i])
            bnd[i + 1].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    ms_total = bnd[0].elapsed_time(bnd[-1])
    step_ms = [bnd[i].elapsed_time(bnd[i + 1]) for i in range(args.steps)]
    kern_ms = [a.elapsed_time(b) for a, b in evs]
    err = ws[:256].view(torch.int32)  # device error word of the fused kernel (first bytes of the workspace)
    ms_step = ms_total / args.steps
    if world > 1:
        t = torch.tensor([ms_step], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_step = float(t.item())

    # end-to-end through the public API with host buffers: H2D of the step's
    # inputs from pinned memory, the call(s), D2H of the gradients.  Sharded: each
    # rank copies its rows of the query-side inputs plus the shared key side and
    # indices, and reads back its dQuery rows and the summed key-side gradients.
    e2e = None
    if not args.no_e2e:
        qside = [p.q, p.q_rope, p.dout, out, smax, ssum]
        shared = [p.k, p.k_rope, p.indices] + ([p.seqlens_q] if p.seqlens_q is not None else [])
        rows = lambda x: x.reshape(T1, -1)[rb:re_]  # this rank's query rows of a [.., T1-row] tensor
        host_q = [rows(x).cpu().pin_memory() for x in qside]
        host_s = [x.cpu().pin_memory() for x in shared]
        dev_q = [torch.zeros_like(x) for x in qside]
        dev_s = [torch.empty_like(x) for x in shared]
        dq, dk, dv, dqr, dkr = outs
        host_out = [torch.empty_like(rows(dq), device="cpu").pin_memory(),
                    torch.empty_like(rows(dqr), device="cpu").pin_memory()] + \
                   [torch.empty_like(x, device="cpu").pin_memory() for x in (dk, dv, dkr)]
        h2d = sum(x.numel() * x.element_size() for x in host_q + host_s)
        d2h = sum(x.numel() * x.element_size() for x in host_out)

        def e2e_step():
            for d, h in zip(dev_q, host_q):
                rows(d).copy_(h, non_blocking=True)
            for d, h in zip(dev_s, host_s):
                d.copy_(h, non_blocking=True)
            q, qr, do, o, mx, sm = dev_q
            k, kr, idx = dev_s[:3]
            sq = dev_s[3] if len(dev_s) > 3 else None
            grad(q, k, idx, do, o, mx, sm, qr, kr, sq, sq)
            for h, o2 in zip(host_out, (rows(dq), rows(dqr), dk, dv, dkr)):
                h.copy_(o2, non_blocking=True)

        if not sharded:
            # one GPU: the library's pipelined host API (chunked rows, copies overlapped with the kernels)
            pl = S.HostPipeline(dev)
            host_all = {n: x.cpu().pin_memory() for n, x in (("q", p.q), ("qr", p.q_rope), ("k", p.k),
                                                             ("kr", p.k_rope), ("do", p.dout), ("o", out),
                                                             ("mx", smax), ("sm", ssum), ("idx", p.indices))}
            host_sq = p.seqlens_q.cpu().pin_memory() if p.seqlens_q is not None else None
            host_res = tuple(torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
                             for x in (p.q, p.k, p.k, p.q_rope, p.k_rope))
            h2d = sum(x.numel() * x.element_size() for x in host_all.values()) + \
                (host_sq.numel() * host_sq.element_size() if host_sq is not None else 0)
            d2h = sum(x.numel() * x.element_size() for x in host_res)

            def e2e_step():
                h = host_all
                S.sfa_grad_host(h["q"], h["k"], True, h["idx"], h["do"], h["o"], h["mx"], h["sm"], h["qr"], h["kr"],
                                scale=p.scale, sparse_block_size=p.block_size, layout=p.layout,
                                sparse_mode=p.sparse_mode, deterministic=p.deterministic,
                                actual_seq_lengths_q=host_sq, actual_seq_lengths_kv=host_sq, outputs=host_res,
                                pipeline=pl, device=dev)

        e2e_step()
        torch.cuda.synchronize(dev)
        n_e2e = max(2, min(args.steps, 5))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        a.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = a.elapsed_time(b) / n_e2e
        if world > 1:
            t = torch.tensor([e2e_ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e_ms = float(t.item())
        e2e = {"value": flop / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    err_word = int(err[0].item())
    return dict(flop=flop, flop_rank=flop_rank, triples=triples, ms_step=ms_step, kern_ms=kern_ms, step_ms=step_ms,
                clocks=clk.summary(), e2e=e2e, ws_bytes=ws_bytes, err_word=err_word, p=p, sharded=sharded,
                rows=(rb, re_), paired=paired)


def run_fwd(args, local_rank):
    """The forward of a sparse workload (sfa_fwd), one GPU: 2176 FLOP per valid
    (row, head, key) triple (S = Q~.K~^T over 576 dims, out = P.V over 512)."""
    import torch
    import sparse_attention_backward_sfa_b200 as S
    from sparse_attention_backward_sfa_b200 import _native as N
    from workloads import WORKLOADS

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    lib = N.load()
    p = build_problem(args.workload, 0, dev)
    _, _, nr = S.compact_indices(p.indices, p.k, p.q, p.q_rope, sparse_block_size=p.block_size, layout=p.layout,
                                 sparse_mode=p.sparse_mode, actual_seq_lengths_q=p.seqlens_q,
                                 actual_seq_lengths_kv=p.seqlens_kv)
    triples = int(nr.to(torch.int64).sum().item()) * p.N1
    flop = triples * 2176
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            N.check(lib.sfa_set_kernel_events(ctypes_ptr(ev[0]), ctypes_ptr(ev[1])))
        S.sfa_fwd(p.q, p.k, p.k, p.indices, p.q_rope, p.k_rope, **kw(p))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in evs:
        a.record(stream)
        b.record(stream)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        torch.cuda.synchronize(dev)
        t0.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
    ms_step = t0.elapsed_time(t1) / args.steps
    kern = statistics.mean(a.elapsed_time(b) for a, b in evs)
    peaks, src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    return {"metric": "sparse-attn forward TFLOP/s (bf16, S + P.V count, 2176 FLOP per triple)",
            "value": flop / (ms_step * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOADS[args.workload], "N1": p.N1, "valid_triples": triples,
                       "path": "tcgen05 (N1 = 128)" if p.N1 == 128 else "CUDA-core"},
            "roofline": {"bound": "tensor", "achieved": flop / (kern * 1e-3) / 1e12, "peak": peak, "unit": "TFLOP/s",
                         "frac": flop / (kern * 1e-3) / 1e12 / peak, "kernel_ms": kern,
                         "traffic": recorded_traffic("fwd4") if args.workload == 4 and not args.seqs else None},
            # fused path: compact, order, block sort (block-sparse, topk <= 4096), expand, fused forward
            "gpu_launches": ((4 + int(p.block_size > 1 and p.topk <= 4096)) if p.N1 == 128 else 2) * args.steps,
            "clocks": clk.summary()}


def indexer_flop_per_pair(N1: int, G: int, Di: int) -> int:
    """Algorithmic FLOP of the indexer gradient per visible (query row, key) pair:
    the main scores (2*N1*576) and the indexer's three contractions (scores, dq~I, dK~I)."""
    return 2 * N1 * 576 + 6 * G * Di


def indexer_inputs(dev, seqs=None):
    """The indexer-gradient workload with consistent statistics: the main attention's
    from sfa_fwd over every causal block, the indexer's max / sum of exp(I - max) over
    the visible keys computed with torch in row chunks (input preparation)."""
    import torch
    import sparse_attention_backward_sfa_b200 as S
    from workloads import make_device_indexer_problem
    p = make_device_indexer_problem(device=dev, **({"seqs": seqs} if seqs else {}))
    lens = np.diff(np.concatenate([[0], p.seqlens_q.cpu().numpy()])).astype(np.int64)
    bs = 16
    nb = int(-(-lens.max() // bs))
    cu32 = p.seqlens_q.to(torch.int32)
    idx = torch.arange(nb, dtype=torch.int32, device=dev).repeat(p.T1, 1).reshape(p.T1, 1, nb).contiguous()
    _, smax, ssum = S.sfa_fwd(p.q, p.k, p.k, idx, p.q_rope, p.k_rope, scale=p.scale, sparse_block_size=bs,
                              layout="TND", sparse_mode=3, actual_seq_lengths_q=cu32, actual_seq_lengths_kv=cu32)
    del idx
    mi = torch.zeros(p.T1, dtype=torch.float32, device=dev)
    li = torch.zeros(p.T1, dtype=torch.float32, device=dev)
    ki = p.k_index.reshape(p.T2, p.Di).float()
    start = 0
    for L in lens.tolist():
        kseq = ki[start:start + L]
        for r0 in range(0, L, 256):
            r1 = min(L, r0 + 256)
            qi = p.q_index[start + r0:start + r1].float()                      # [r, G, Di]
            w = p.weights[start + r0:start + r1].float()                       # [r, G]
            I = torch.einsum("rg,rgj->rj", w, torch.relu(torch.einsum("rgd,jd->rgj", qi, kseq)))
            pos = torch.arange(r0, r1, device=dev)[:, None]
            I = I.masked_fill(torch.arange(L, device=dev)[None, :] > pos, float("-inf"))
            m = I.max(dim=1).values
            mi[start + r0:start + r1] = m
            li[start + r0:start + r1] = torch.exp(I - m[:, None]).sum(dim=1)
        start += L
    return p, lens, smax, ssum, mi, li


def run_indexer(args, local_rank):
    """The dense lightning-indexer gradient with KL loss (lig_kl_grad), one GPU, TND
    sequences {2048, 4096, 4096, 6144}, N1 = 128, G = 64, Di = 128, causal."""
    import torch
    import sparse_attention_backward_sfa_b200 as S
    from sparse_attention_backward_sfa_b200 import _native as N

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    lib = N.load()
    p, lens, smax, ssum, mi, li = indexer_inputs(dev, SEQS if args.seqs else None)
    pairs = int(sum(int(L) * (int(L) + 1) // 2 for L in lens))
    flop = pairs * indexer_flop_per_pair(p.N1, p.G, p.Di)
    shape = S.lig_shape(p.q, p.k, p.q_index, p.k_index, "TND", p.seqlens_q)
    ws = torch.empty(S.lig_kl_grad_workspace_size(shape, 3), dtype=torch.uint8, device=dev)
    outs = (torch.empty_like(p.q_index), torch.empty_like(p.k_index), torch.empty_like(p.weights),
            torch.empty(1, dtype=torch.float32, device=dev))
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            N.check(lib.sfa_set_kernel_events(ctypes_ptr(ev[0]), ctypes_ptr(ev[1])))
        S.lig_kl_grad(p.q, p.k, p.q_index, p.k_index, p.weights, smax, ssum, mi, li, p.q_rope, p.k_rope,
                      scale=p.scale, layout="TND", sparse_mode=3, actual_seq_lengths_query=p.seqlens_q,
                      actual_seq_lengths_key=p.seqlens_kv, workspace=ws, outputs=outs)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in evs:
        a.record(stream)
        b.record(stream)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        torch.cuda.synchronize(dev)
        t0.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
    ms_step = t0.elapsed_time(t1) / args.steps
    kern = statistics.mean(a.elapsed_time(b) for a, b in evs)
    err = int(ws[:4].view(torch.int32).item())
    peaks, src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    e2e = None
    if not args.no_e2e:
        e2e = indexer_e2e(p, smax, ssum, mi, li, ws, args)
    cpu = None
    if not args.no_cpu_baseline:
        cpu = indexer_cpu_baseline(p, lens, smax, ssum, mi, li, args.cpu_budget)
    from workloads import INDEXER_WORKLOAD
    if e2e is not None:
        e2e = {"value": flop / (e2e["ms_per_step"] * 1e-3) / 1e12, "unit": "TFLOP/s", **e2e}
    return {"metric": "lightning-indexer KL-loss backward TFLOP/s (bf16, 2*N1*576 + 6*G*Di FLOP per visible pair)",
            "value": flop / (ms_step * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": INDEXER_WORKLOAD if not args.seqs else f"indexer_kl_tnd_{args.seqs}",
                       "N1": p.N1, "G": p.G, "Di": p.Di, "visible_pairs": pairs,
                       "l2": "inputs larger than L2 (q 2.4 GB per step)"},
            "roofline": {"bound": "tensor", "achieved": flop / (kern * 1e-3) / 1e12, "peak": peak, "unit": "TFLOP/s",
                         "frac": flop / (kern * 1e-3) / 1e12 / peak, "kernel": "lig_fused_kernel", "kernel_ms": kern,
                         "peak_source": src,
                         "traffic": recorded_traffic("lig") if not args.seqs else None},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": 7 * args.steps, "clocks": clk.summary(),
            "device_error_word": err}


def indexer_e2e(p, smax, ssum, mi, li, ws, args):
    """The same call end to end: every step copies its inputs from pinned host memory to the
    device, runs lig_kl_grad and copies the four results back, all inside the timed region."""
    import torch
    import sparse_attention_backward_sfa_b200 as S
    dev = p.q.device
    names = ("q", "k", "q_index", "k_index", "weights", "q_rope", "k_rope")
    host_in = {n: getattr(p, n).cpu().pin_memory() for n in names}
    host_st = [x.cpu().pin_memory() for x in (smax, ssum, mi, li)]
    dev_in = {n: torch.empty_like(getattr(p, n)) for n in names}
    dev_st = [torch.empty_like(x) for x in (smax, ssum, mi, li)]
    outs = (torch.empty_like(p.q_index), torch.empty_like(p.k_index), torch.empty_like(p.weights),
            torch.empty(1, dtype=torch.float32, device=dev))
    host_out = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
    h2d = sum(x.numel() * x.element_size() for x in list(host_in.values()) + host_st)
    d2h = sum(o.numel() * o.element_size() for o in outs)

    def step():
        for n in names:
            dev_in[n].copy_(host_in[n], non_blocking=True)
        for d, h in zip(dev_st, host_st):
            d.copy_(h, non_blocking=True)
        S.lig_kl_grad(dev_in["q"], dev_in["k"], dev_in["q_index"], dev_in["k_index"], dev_in["weights"], *dev_st,
                      dev_in["q_rope"], dev_in["k_rope"], scale=p.scale, layout="TND", sparse_mode=3,
                      actual_seq_lengths_query=p.seqlens_q, actual_seq_lengths_key=p.seqlens_kv, workspace=ws,
                      outputs=outs)
        for h, o in zip(host_out, outs):
            h.copy_(o, non_blocking=True)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    ms = t0.elapsed_time(t1) / args.steps
    return {"ms_per_step": ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


def indexer_cpu_baseline(p, lens, smax, ssum, mi, li, budget_s: float):
    """The indexer oracle (fp64 numpy, as it stands) on a bounded sample of query rows."""
    import torch
    from oracle import indexer_kl_oracle as O
    from workloads import RowView
    rng = np.random.default_rng(54321)
    T1 = p.T1
    k = p.k.reshape(p.T2, p.D).float().cpu().numpy()
    kr = p.k_rope.reshape(p.T2, p.Dr).float().cpu().numpy()
    ki = p.k_index.reshape(p.T2, p.Di).float().cpu().numpy()
    sq = p.seqlens_q.cpu().numpy()
    starts = np.concatenate([[0], sq[:-1]])
    per_pair = indexer_flop_per_pair(p.N1, p.G, p.Di)
    done, elapsed, flop, n = 0, 0.0, 0, 2
    while elapsed < budget_s and done < T1:
        toks = np.sort(rng.choice(T1, size=n, replace=False))
        views = [RowView(x, toks, T1) for x in (p.q, p.q_rope, p.q_index, p.weights, smax, ssum, mi.reshape(T1, 1),
                                                li.reshape(T1, 1))]
        qv, qrv, qiv, wv, mv, lv, miv, liv = views
        c0 = time.perf_counter()
        O.indexer_kl_grad(qv, k, qiv, ki, wv, mv, lv, miv, liv, qrv, kr, p.scale, "TND", p.B, 0, 0, sq, sq, 3,
                          tokens=toks)
        elapsed += time.perf_counter() - c0
        for t in toks:
            b = int(np.searchsorted(sq, t, side="right"))
            flop += (int(t) - int(starts[b]) + 1) * per_pair
        done += n
        n = min(2 * n, 64)
    return {"value": flop / elapsed / 1e12 if elapsed > 0 else 0.0, "unit": "TFLOP/s",
            "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
            "sample": f"{done} query rows of the indexer workload (fp64 numpy oracle, {elapsed:.1f} s)"}


def run_fa(args, rank, world, local_rank):
    """Workload 2: dense varlen FA backward (TND, causal); 1280 FLOP per valid
    (query row, head, key) triple."""
    import torch
    import torch.distributed as dist
    import sparse_attention_backward_sfa_b200 as S
    from sparse_attention_backward_sfa_b200 import _native as N
    from workloads import make_fa_problem

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    lib = N.load()
    fp = make_fa_problem(seed=1002 + 7919 * rank, D=args.fa_d)
    t = lambda a: torch.from_numpy(a).to(device=dev, dtype=torch.bfloat16)
    q, k, v, dy = t(fp.q), t(fp.k), t(fp.v), t(fp.dy)
    out, smax, ssum = S.fa_fwd(q, k, v, fp.cu_seqlens_q, fp.cu_seqlens_kv, scale=fp.scale, sparse_mode=3)
    lens = np.diff(np.concatenate([[0], fp.cu_seqlens_q]))
    triples = int(sum(L * (L + 1) // 2 for L in lens)) * fp.Nq
    flop = triples * 10 * fp.D  # five GEMMs of 2*D FLOP per triple (1280 at D = 128)
    outs = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            N.check(lib.sfa_set_kernel_events(ctypes_ptr(ev[0]), ctypes_ptr(ev[1])))
        S.fa_grad(q, k, v, dy, smax, ssum, out, fp.cu_seqlens_q, fp.cu_seqlens_kv, scale=fp.scale, sparse_mode=3,
                  outputs=outs)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in evs:
        a.record(stream)
        b.record(stream)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        torch.cuda.synchronize(dev)
        t0.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
    ms_step = t0.elapsed_time(t1) / args.steps
    if world > 1:
        tt = torch.tensor([ms_step], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms_step = float(tt.item())
    kern_ms = [a.elapsed_time(b) for a, b in evs]
    return dict(flop=flop, triples=triples, ms_step=ms_step, kern_ms=kern_ms, clocks=clk.summary(), e2e=None,
                ws_bytes=0, err_word=0, p=None)


def ctypes_ptr(ev):
    import ctypes
    return ctypes.c_void_p(ev.cuda_event)


class _SampledRows:
    """Row access t -> the oracle forward's output row for a sorted sample of query rows."""

    def __init__(self, arr, toks, n):
        self._rows = {int(t): arr[i] for i, t in enumerate(toks)}
        self._n = n

    def __len__(self):
        return self._n

    def __getitem__(self, t):
        return self._rows[int(t)]


def cpu_baseline(workload: int, budget_s: float):
    """Time the oracle (fp64 numpy, as it stands) on a bounded sample of query
    rows of the same workload on this host's cores.  O and the softmax statistics
    of the sampled rows come from the oracle's own forward (input preparation,
    not timed), so this arm runs no code of the library."""
    import torch
    from oracle import sfa_oracle as O
    from workloads import RowView
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    p = build_problem(workload, 0, dev)
    rng = np.random.default_rng(12345)
    T1 = p.T1
    k = p.k.reshape(p.T2, p.D).float().cpu().numpy()
    kr = p.k_rope.reshape(p.T2, p.Dr).float().cpu().numpy()
    sq = None if p.seqlens_q is None else p.seqlens_q.cpu().numpy()
    done_tokens, elapsed, flop = 0, 0.0, 0
    n = 2
    while elapsed < budget_s and done_tokens < T1:
        toks = np.sort(rng.choice(T1, size=n, replace=False))
        qv, qrv, dov, iv = (RowView(x, toks, T1) for x in (p.q, p.q_rope, p.dout, p.indices))
        out, m, l = O.sfa_forward(qv, k, k, iv, qrv, kr, p.scale, p.block_size, p.sparse_mode, p.layout, p.B, p.S1,
                                  p.S2, sq, sq, tokens=toks)
        ov, mv, lv = (_SampledRows(a, toks, T1) for a in (out, m, l))
        c0 = time.perf_counter()
        O.sfa_backward(qv, k, k, iv, dov, ov, mv, lv, qrv, kr, p.scale, p.block_size, p.sparse_mode, p.layout,
                       p.B, p.S1, p.S2, sq, sq, tokens=toks)
        elapsed += time.perf_counter() - c0
        for t in toks:
            nrow = 0
            row = iv[t]
            # rows of this token (same rule as the oracle)
            sp = [s for s in O.make_spans(p.layout, p.B, p.S1, p.S2, sq, sq) if s.q_start <= t < s.q_start + s.q_len]
            if sp:
                s = sp[0]
                nrow = len(O.selected_rows(np.asarray(row).ravel(), p.block_size, int(t) - s.q_start, s.q_len,
                                           s.kv_len, p.sparse_mode))
            flop += nrow * p.N1 * FLOP_PER_TRIPLE
        done_tokens += n
        n = min(2 * n, 64)
    cores = len(os.sched_getaffinity(0))
    return {"value": flop / elapsed / 1e12 if elapsed > 0 else 0.0, "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle", "sample": f"{done_tokens} query rows of workload {workload} "
                                        f"(fp64 numpy oracle, {elapsed:.1f} s; O and statistics of those rows "
                                        f"from the oracle forward, not timed)", "seconds": elapsed}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", type=int, default=4, choices=[2, 3, 4, 5])
    ap.add_argument("--fa-d", type=int, default=128, help="workload 2: head dim (128 as configured; 64 a variant)")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--fwd", action="store_true",
                    help="time the forward (sfa_fwd: out + softmax statistics) instead of the backward")
    ap.add_argument("--indexer", action="store_true",
                    help="time the dense lightning-indexer gradient with KL loss (lig_kl_grad)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seqs", default=None,
                    help="smaller profiling case: comma-separated sequence lengths replacing workload 4's, "
                         "or workload 5's sequence length (topk scaled with it)")
    args = ap.parse_args()
    global SEQS
    if args.seqs:
        SEQS = [int(x) for x in args.seqs.split(",")]
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    from workloads import WORKLOADS

    if args.impl == "reference":
        if rank != 0:
            return
        per_step = []
        res = None
        budget = max(2.0, min(20.0, 90.0 / max(1, args.steps)))  # whole run ~1.5-2 min
        for i in range(args.warmup + args.steps):
            res = cpu_baseline(args.workload, budget if i >= args.warmup else 1.0)
            if i >= args.warmup:
                per_step.append(res)
        val = statistics.mean(r["value"] for r in per_step)
        line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": 1,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": statistics.mean(r["seconds"] for r in per_step) * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": WORKLOADS[args.workload], "sample": per_step[-1]["sample"]},
                "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": per_step[-1]["cores"], "kind": "oracle",
                                 "sample": per_step[-1]["sample"]},
                "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    from datetime import timedelta
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    if args.indexer:
        if world > 1:
            raise SystemExit("--indexer: one GPU")
        print(json.dumps(run_indexer(args, local_rank)), flush=True)
        return
    if args.fwd:
        if world > 1 or args.workload == 2:
            raise SystemExit("--fwd: one GPU, sparse workloads (3, 4, 5)")
        print(json.dumps(run_fwd(args, local_rank)), flush=True)
        return
    r = run_fa(args, rank, world, local_rank) if args.workload == 2 else run_ours(args, rank, world, local_rank)
    peaks, src = load_peaks()
    sharded = bool(r.get("sharded"))
    # sharded: r["flop"] is the whole workload, split over the ranks; replicas: per rank
    value = r["flop"] * (1 if sharded else world) / (r["ms_step"] * 1e-3) / 1e12
    kern = statistics.mean(r["kern_ms"])
    achieved = r.get("flop_rank", r["flop"]) / (kern * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.workload != 2:
        cpu = cpu_baseline(args.workload, args.cpu_budget)
        cpu.pop("seconds", None)
    if rank == 0 and args.workload == 2:
        line = {"metric": f"dense varlen FA backward TFLOP/s (bf16, 5-GEMM count, D={args.fa_d})", "value": value,
                "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": r["ms_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": {"workload": WORKLOADS[2] if args.fa_d == 128 else WORKLOADS[2].replace("d128", f"d{args.fa_d}"),
                           "valid_triples": r["triples"], "gflop_per_step": r["flop"] / 1e9},
                "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                             "frac": achieved / peak, "kernel": "fa_bwd_fused_kernel", "kernel_ms": kern,
                             "traffic": recorded_traffic(2) if args.fa_d == 128 else None},
                "gpu_launches": 3 * args.steps, "clocks": r["clocks"]}
        print(json.dumps(line), flush=True)
    elif rank == 0:
        p = r["p"]
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": r["ms_step"],
            "ms_per_step_median": statistics.median(r["step_ms"]),
            "ms_per_step_min_max": [min(r["step_ms"]), max(r["step_ms"])], "higher_is_better": True,
            "scaling": "strong" if sharded else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "pct_of_peak": 100.0 * value / world / peak,
            "config": {"workload": WORKLOADS[args.workload] + (f" seqs={args.seqs}" if args.seqs else ""),
                       "layout": p.layout, "N1": p.N1, "topk": p.topk,
                       "sparse_block_size": p.block_size, "deterministic": p.deterministic,
                       "valid_triples": r["triples"], "gflop_per_step": r["flop"] / 1e9,
                       "l2": "inputs larger than L2 (q+dO+O %.1f GB per step)" % (3 * p.q.numel() * 2 / 1e9),
                       "parallelism": (f"query rows sharded over {world} GPUs by work, NCCL all-reduce of the "
                                       f"dK/dV accumulator" if sharded else "single GPU")},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "peak_source": f"{src} bf16 burst",
                         "peak_sustained": float(peaks.get("bf16_tflops_sustained", peak)),
                         "frac_sustained": achieved / float(peaks.get("bf16_tflops_sustained", peak)),
                         # the events bracket both backward launches (paired rows, then the rest);
                         # the kernel named is the one that takes most of the work
                         "kernel": "sfa_bwd_pair_kernel" if r["paired"] >= 0.5 else "sfa_bwd_fused_kernel",
                         "paired_work_fraction": r["paired"],
                         "kernel_ms": kern,
                         "kernel_ms_median": statistics.median(r["kern_ms"]),
                         "traffic": recorded_traffic(args.workload) if not args.seqs and not sharded else None},
            "cpu_baseline": cpu,
            "e2e": r["e2e"],
            # compact, rowsum, order, block sort (block-sparse lists of topk <= 4096), expand, [N1 = 128:
            # pair flags, pair lists, paired kernel], single-row kernel, cast
            "gpu_launches": (6 + int(p.block_size > 1 and p.topk <= 4096) + (3 if p.N1 == 128 else 0)) * args.steps,
            "clocks": r["clocks"],
            "device_error_word": r["err_word"],
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
