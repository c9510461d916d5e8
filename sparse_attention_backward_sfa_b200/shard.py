"""Query-row sharding of the sparse attention backward over several GPUs.

Each rank owns a contiguous range of query rows (the flattened [T1] row index),
runs the backward of those rows (sfa_grad_rows) with the full key / value
replicated, and the ranks then sum their key-side accumulators with one
all-reduce: dKey, dKeyRope and dValue are sums over every query row that
selected a key (SparseFlashAttentionGrad README, 功能说明), so partial sums over
disjoint row sets add up to the whole.  dQuery rows stay on the rank that owns
them.  In deterministic mode the accumulator is int64 fixed point on a grid set
by max|dOut| over all ranks' rows (one max all-reduce of a single float first),
so the sum all-reduce is exact and the result does not depend on the rank count
or order.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import numpy as np

Range = Tuple[int, int]


def balanced_row_ranges(row_work: Sequence[float], parts: int, align: int = 2) -> List[Range]:
    """Splits rows 0..len(row_work) into `parts` contiguous ranges of about equal total work.

    Boundary k sits at the row edge whose cumulative work is closest to k/parts of the
    total (the last range ends at the last row), rounded to a multiple of `align`: the
    backward processes rows (2m, 2m + 1) with identical block lists as one pair, so
    even boundaries keep every pair of the whole call together (deterministic results
    then equal the unsharded call bit for bit).  Ranges may be empty when rows are few
    or work is concentrated.
    """
    if parts < 1:
        raise ValueError("parts must be >= 1")
    if align < 1:
        raise ValueError("align must be >= 1")
    w = np.asarray(row_work, dtype=np.float64)
    if w.ndim != 1 or (w.size and w.min() < 0):
        raise ValueError("row_work must be a 1-D sequence of non-negative numbers")
    n = w.size
    cum = np.cumsum(w)
    total = float(cum[-1]) if n else 0.0
    bounds = [0]
    for k in range(1, parts):
        if total > 0:
            target = total * k / parts
            i = int(np.searchsorted(cum, target, side="left"))  # first row reaching the target
            hi = min(i + 1, n)                                   # edge after that row
            lo = i                                               # edge before it
            b = lo if lo > 0 and target - cum[lo - 1] <= cum[hi - 1] - target else hi
        else:
            b = (n * k) // parts
        b = int(round(b / align)) * align
        bounds.append(min(max(b, bounds[-1]), n))
    bounds.append(n)
    return [(bounds[k], bounds[k + 1]) for k in range(parts)]


def row_work(nrows) -> np.ndarray:
    """Per-row work weight: the row's number of valid key rows (its (row, key) pairs)."""
    return np.asarray(nrows, dtype=np.float64)


def sfa_grad_sharded(query, key, value, sparse_indices, d_out, out, softmax_max, softmax_sum, query_rope, key_rope,
                     *, scale: float, sparse_block_size: int, layout: str, sparse_mode: int,
                     deterministic: bool = False, actual_seq_lengths_q=None, actual_seq_lengths_kv=None,
                     group=None, ranges: Optional[List[Range]] = None, workspace=None, dkv_accum=None,
                     outputs=None, stream=None):
    """Sharded backward on the calling rank of `group` (torch.distributed; NCCL for CUDA tensors).

    Every rank passes the same full tensors.  Returns (dQuery, dKey, dValue, dQueryRope, dKeyRope,
    (row_begin, row_end)): the dQuery / dQueryRope rows of this rank's range (other rows are left as
    they were in `outputs`, zero when allocated here) and the complete key-side gradients, identical
    on every rank.  `ranges` (one per rank) defaults to a work-balanced split computed from the
    index compaction (one device-to-host copy of the per-row counts).
    """
    import torch
    import torch.distributed as dist

    from . import ops

    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    kw = dict(layout=layout, actual_seq_lengths_q=actual_seq_lengths_q)
    if ranges is None:
        _, _, nr = ops.compact_indices(sparse_indices, key, query, query_rope, sparse_block_size=sparse_block_size,
                                       sparse_mode=sparse_mode, actual_seq_lengths_kv=actual_seq_lengths_kv,
                                       stream=stream, **kw)
        ranges = balanced_row_ranges(row_work(nr.cpu().numpy()), world)
    if len(ranges) != world:
        raise ValueError(f"{len(ranges)} ranges for {world} ranks")
    rb, re_ = ranges[rank]
    if dkv_accum is None:
        dkv_accum = ops.sfa_dkv_accumulator(query, key, query_rope, sparse_indices, deterministic=deterministic, **kw)
    else:
        dkv_accum.zero_()
    if outputs is None:
        outputs = (torch.zeros_like(query), None, None, torch.zeros_like(query_rope), None)
    dq, dk, dv, dqr, dkr = outputs
    dmax = None
    if deterministic:
        # the fixed-point grid follows max|dOut| over ALL ranks' rows: every rank must use the same one
        dmax = ops.dout_absmax(d_out, query, key, query_rope, sparse_indices, row_begin=rb, row_end=re_,
                               stream=stream, **kw)
        if world > 1:
            dist.all_reduce(dmax, op=dist.ReduceOp.MAX, group=group)
    ops.sfa_grad_rows(query, key, value, sparse_indices, d_out, out, softmax_max, softmax_sum, query_rope, key_rope,
                      row_begin=rb, row_end=re_, dkv_accum=dkv_accum, scale=scale,
                      sparse_block_size=sparse_block_size, sparse_mode=sparse_mode, deterministic=deterministic,
                      dout_absmax=dmax, actual_seq_lengths_kv=actual_seq_lengths_kv, workspace=workspace,
                      d_query=dq, d_query_rope=dqr, stream=stream, **kw)
    if world > 1:
        dist.all_reduce(dkv_accum, op=dist.ReduceOp.SUM, group=group)
    key_outs = None if dk is None else (dk, dv, dkr)
    dk, dv, dkr = ops.sfa_dkv_finalize(dkv_accum, query, key, query_rope, sparse_indices,
                                       deterministic=deterministic, dout_absmax=dmax, scale=scale, outputs=key_outs,
                                       stream=stream, **kw)
    return dq, dk, dv, dqr, dkr, (rb, re_)
