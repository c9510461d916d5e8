"""Sparse attention backward for host-resident (pinned) tensors, with the copies
overlapped with the computation.

The query rows are processed in chunks (sfa_grad_rows), last rows first: while one chunk runs
on the compute stream, the next chunk's query-side inputs (query, queryRope, dOut, out,
softmax statistics, sparse indices) are copied host->device on a copy stream and the previous
chunk's dQuery / dQueryRope rows are copied device->host on a third stream.  The
key-side inputs go first (in deterministic mode followed by all
of dOut, whose largest magnitude sets the fixed-point grid before the first
chunk runs); the key-side gradients are cast from the accumulator and copied
back at the end.  PCIe is full duplex, so a step
costs about max(H2D time, compute time) plus one chunk of each, instead of
their sum.
"""
from __future__ import annotations

from typing import Dict, Optional

import torch

from . import ops


def _rows(x: torch.Tensor, T1: int, a: int, b: int) -> torch.Tensor:
    """Rows [a, b) of a tensor whose leading dims flatten to T1 query rows."""
    return x.reshape(T1, -1)[a:b]


class HostPipeline:
    """Device buffers, streams and events for repeated sfa_grad_host calls on one shape."""

    def __init__(self, device: torch.device):
        self.device = device
        self.buf: Dict[str, torch.Tensor] = {}
        self.h2d = torch.cuda.Stream(device)
        self.d2h = torch.cuda.Stream(device)

    def _like(self, name: str, x: torch.Tensor, zero: bool = False) -> torch.Tensor:
        t = self.buf.get(name)
        if t is None or t.shape != x.shape or t.dtype != x.dtype:
            t = (torch.zeros if zero else torch.empty)(x.shape, dtype=x.dtype, device=self.device)
            self.buf[name] = t
        return t


def sfa_grad_host(query, key, value_is_key: bool, sparse_indices, d_out, out, softmax_max, softmax_sum, query_rope,
                  key_rope, *, scale: float, sparse_block_size: int, layout: str, sparse_mode: int,
                  deterministic: bool = False, actual_seq_lengths_q=None, actual_seq_lengths_kv=None,
                  outputs=None, chunks: int = 16, pipeline: Optional[HostPipeline] = None, device=None):
    """sfa_grad on pinned host tensors; returns host (dQuery, dKey, dValue, dQueryRope, dKeyRope).

    value == key is the only layout the pages support (`value_is_key` must be True).  `outputs`
    are pinned host tensors to fill (allocated when None).  The copies and kernels are enqueued
    on the current stream of `device` and two side streams; the call returns after the results
    are on the host.
    """
    if not value_is_key:
        raise ValueError("sfa_grad_host: value must be key")
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    pl = pipeline or HostPipeline(dev)
    comp = torch.cuda.current_stream(dev)
    lead = query.shape[:-2]
    T1 = 1
    for d in lead:
        T1 *= d
    # a row range reads only its own rows of these (the indices included), so they go over per chunk
    qside = {"q": query, "qr": query_rope, "do": d_out, "o": out, "mx": softmax_max, "sm": softmax_sum,
             "idx": sparse_indices}
    shared = {"k": key, "kr": key_rope}
    if actual_seq_lengths_q is not None:
        shared["sq"] = actual_seq_lengths_q
    if actual_seq_lengths_kv is not None and actual_seq_lengths_kv is not actual_seq_lengths_q:
        shared["skv"] = actual_seq_lengths_kv
    dq_ = {n: pl._like(n, x, zero=True) for n, x in qside.items()}
    ds_ = {n: pl._like(n, x) for n, x in shared.items()}
    sq = ds_.get("sq")
    skv = ds_.get("skv", sq) if actual_seq_lengths_kv is not None else None
    g_dq = pl._like("g_dq", query)
    g_dqr = pl._like("g_dqr", query_rope)
    g_dk = pl._like("g_dk", key)
    g_dv = pl._like("g_dv", key)
    kr_shape = key_rope
    g_dkr = pl._like("g_dkr", kr_shape)
    kw = dict(layout=layout, actual_seq_lengths_q=sq)
    acc = pl.buf.get("acc")
    if acc is None or acc.dtype != (torch.int64 if deterministic else torch.float32):
        acc = ops.sfa_dkv_accumulator(dq_["q"], ds_["k"], dq_["qr"], dq_["idx"], deterministic=deterministic, **kw)
        pl.buf["acc"] = acc
    ws = pl.buf.get("ws")
    shape = ops.sfa_shape(dq_["q"], ds_["k"], dq_["qr"], dq_["idx"], layout, sq)
    need = ops.sfa_grad_workspace_size(shape, sparse_block_size, sparse_mode, deterministic)
    if ws is None or ws.numel() < need:
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
        pl.buf["ws"] = ws
    if outputs is None:
        outputs = tuple(torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
                        for x in (query, key, key, query_rope, key_rope))
    h_dq, h_dk, h_dv, h_dqr, h_dkr = outputs

    chunks = max(1, min(chunks, T1))
    # chunk boundaries on even rows: rows (2m, 2m + 1) that share their blocks stay one pair, as in
    # the single call (deterministic results are then bit-identical to it)
    bounds = [min(T1, 2 * ((T1 * c) // (2 * chunks))) for c in range(chunks)] + [T1]
    # last rows first: under a causal mask they select the most keys, so the call ends on its
    # lightest chunk (the compute left after the last host->device copy is the smallest)
    order = range(chunks - 1, -1, -1)
    # the copy stream starts after whatever the caller queued before this call
    pl.h2d.wait_stream(comp)
    with torch.cuda.stream(pl.h2d):
        for n, x in shared.items():
            ds_[n].copy_(x, non_blocking=True)
    ev_shared = torch.cuda.Event()
    ev_shared.record(pl.h2d)
    ev_in, ev_out = [], []
    dmax = None
    with torch.cuda.stream(pl.h2d):
        if deterministic:
            # the fixed-point grid follows max|dOut| over every row: dOut goes over first
            dq_["do"].copy_(d_out, non_blocking=True)
            dmax = pl._like("dmax", torch.empty(1, dtype=torch.float32))
            dmax.zero_()
            ops.dout_absmax(dq_["do"], dq_["q"], ds_["k"], dq_["qr"], dq_["idx"], into=dmax, stream=pl.h2d, **kw)
        for c in order:
            a, b = bounds[c], bounds[c + 1]
            for n, x in qside.items():
                if n == "do" and deterministic:
                    continue
                _rows(dq_[n], T1, a, b).copy_(_rows(x, T1, a, b), non_blocking=True)
            e = torch.cuda.Event()
            e.record(pl.h2d)
            ev_in.append(e)
    comp.wait_event(ev_shared)
    acc.zero_()
    pl.d2h.wait_stream(comp)
    for i, c in enumerate(order):
        a, b = bounds[c], bounds[c + 1]
        comp.wait_event(ev_in[i])
        ops.sfa_grad_rows(dq_["q"], ds_["k"], ds_["k"], dq_["idx"], dq_["do"], dq_["o"], dq_["mx"], dq_["sm"],
                          dq_["qr"], ds_["kr"], row_begin=a, row_end=b, dkv_accum=acc, scale=scale,
                          sparse_block_size=sparse_block_size, sparse_mode=sparse_mode, deterministic=deterministic,
                          dout_absmax=dmax, actual_seq_lengths_kv=skv, workspace=ws, d_query=g_dq,
                          d_query_rope=g_dqr, stream=comp, **kw)
        e = torch.cuda.Event()
        e.record(comp)
        ev_out.append(e)
        pl.d2h.wait_event(e)
        with torch.cuda.stream(pl.d2h):
            _rows(h_dq, T1, a, b).copy_(_rows(g_dq, T1, a, b), non_blocking=True)
            _rows(h_dqr, T1, a, b).copy_(_rows(g_dqr, T1, a, b), non_blocking=True)
    ops.sfa_dkv_finalize(acc, dq_["q"], ds_["k"], dq_["qr"], dq_["idx"], deterministic=deterministic,
                         dout_absmax=dmax, scale=scale, outputs=(g_dk, g_dv, g_dkr), stream=comp, **kw)
    pl.d2h.wait_stream(comp)
    with torch.cuda.stream(pl.d2h):
        h_dk.copy_(g_dk, non_blocking=True)
        h_dv.copy_(g_dv, non_blocking=True)
        h_dkr.copy_(g_dkr, non_blocking=True)
    comp.wait_stream(pl.d2h)
    comp.synchronize()
    return h_dq, h_dk, h_dv, h_dqr, h_dkr
