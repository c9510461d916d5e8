"""PyTorch-facing binding of libsfa: argument marshalling only.

Tensors supply device memory and the current CUDA stream; every step of the
computation runs in the library's kernels.  Each function mirrors the C entry
point of the same name in include/sfa.h.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import numpy as np
import torch

from . import _native as N

_DT = {torch.bfloat16: N.DTYPE_BF16, torch.float16: N.DTYPE_FP16}
ACC_WIDTH = 1088  # key-side accumulator row: dKey 512 | dKeyRope 64 | dValue 512


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(cond: bool, msg: str):
    if not cond:
        raise ValueError(msg)


def _check16(name, t, dtype):
    _need(t.is_contiguous(), f"{name} must be contiguous")
    _need(t.dtype == dtype, f"{name} must be {dtype}")


def _check_cuda(named):
    """Device placement, checked after every size check (so a wrong size is reported as such)."""
    for name, t in named:
        if t is not None:
            _need(t.is_cuda, f"{name} must be a CUDA tensor")


def _check_numel(items):
    """The library reads raw pointers: every tensor must hold exactly the elements its layout implies."""
    for name, t, n in items:
        if t is not None:
            _need(t.numel() == n, f"{name}: {t.numel()} elements, expected {n}")


def _check_f32(name, t):
    _need(t.is_contiguous() and t.dtype == torch.float32, f"{name}: contiguous fp32 tensor")


def _check_outputs(outputs, likes):
    """Caller-supplied outputs: CUDA, contiguous, the dtype and element count of the tensor each mirrors."""
    for (name, t), like in zip(outputs, likes):
        if t is None:
            continue
        _need(t.is_contiguous(), f"{name} must be contiguous")
        _need(t.dtype == like[0], f"{name} must be {like[0]}")
        _need(t.numel() == like[1], f"{name}: {t.numel()} elements, expected {like[1]}")
        _need(t.is_cuda, f"{name} must be a CUDA tensor")


def _check_sfa_inputs(shape, query, key, value, sparse_indices, query_rope, key_rope, d_out=None, out=None,
                      softmax_max=None, softmax_sum=None):
    """Element counts of the sparse attention inputs against the sizes derived from `shape`."""
    T1, T2, N1, N2, D, Dr = shape.T1, shape.T2, shape.N1, shape.N2, shape.D, shape.Dr
    _need(sparse_indices.dtype == torch.int32 and sparse_indices.is_contiguous(),
          "sparse_indices: int32 contiguous tensor")
    for name, t in (("softmax_max", softmax_max), ("softmax_sum", softmax_sum)):
        if t is not None:
            _check_f32(name, t)
    _check_numel((("key", key, T2 * N2 * D), ("value", value, T2 * N2 * D), ("key_rope", key_rope, T2 * N2 * Dr),
                  ("query_rope", query_rope, T1 * N1 * Dr), ("sparse_indices", sparse_indices, T1 * N2 * shape.topk),
                  ("d_out", d_out, T1 * N1 * D), ("out", out, T1 * N1 * D), ("softmax_max", softmax_max, T1 * N1),
                  ("softmax_sum", softmax_sum, T1 * N1)))


def _sfa_named(query, key, value, sparse_indices, query_rope, key_rope, d_out=None, out=None, softmax_max=None,
               softmax_sum=None):
    return (("query", query), ("key", key), ("value", value), ("sparse_indices", sparse_indices),
            ("query_rope", query_rope), ("key_rope", key_rope), ("d_out", d_out), ("out", out),
            ("softmax_max", softmax_max), ("softmax_sum", softmax_sum))


def sfa_shape(query: torch.Tensor, key: torch.Tensor, query_rope: torch.Tensor, sparse_indices: torch.Tensor,
              layout: str, actual_seq_lengths_q=None) -> N.SfaShape:
    s = N.SfaShape()
    _need(query.dtype in _DT, "query must be bf16 or fp16")
    s.dtype = _DT[query.dtype]
    if layout == "BSND":
        _need(query.dim() == 4 and key.dim() == 4, "BSND tensors are 4-D")
        s.layout = N.LAYOUT_BSND
        s.B, s.S1, s.N1, s.D = query.shape
        _, s.S2, s.N2, _ = key.shape
        s.T1, s.T2 = s.B * s.S1, s.B * s.S2
    elif layout == "TND":
        _need(query.dim() == 3 and key.dim() == 3, "TND tensors are 3-D")
        s.layout = N.LAYOUT_TND
        s.T1, s.N1, s.D = query.shape
        s.T2, s.N2, _ = key.shape
        s.S1 = s.S2 = 0
        _need(actual_seq_lengths_q is not None, "TND needs actual sequence lengths")
        s.B = actual_seq_lengths_q.numel()
    else:
        raise ValueError(f"layout {layout!r}")
    s.Dr = query_rope.shape[-1]
    s.topk = sparse_indices.shape[-1]
    return s


def _seqlens(x, layout, B):
    if x is None:
        _need(layout == "BSND", "TND needs actual sequence lengths")
        return None
    _need(x.is_cuda and x.dtype == torch.int32 and x.numel() == B, "seq lengths: int32 CUDA tensor of length B")
    return x


def _workspace(workspace, nbytes: int, device):
    """The caller's workspace (a contiguous uint8 CUDA tensor of at least `nbytes`), or a new one."""
    if workspace is None:
        return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)
    _need(workspace.is_cuda and workspace.is_contiguous() and workspace.dtype == torch.uint8,
          "workspace: contiguous uint8 CUDA tensor")
    _need(workspace.numel() >= nbytes, f"workspace: {workspace.numel()} bytes, need {nbytes}")
    return workspace


def sfa_grad_workspace_size(shape: N.SfaShape, sparse_block_size: int, sparse_mode: int, deterministic: bool) -> int:
    lib = N.load()
    n = ctypes.c_size_t()
    N.check(lib.sfa_grad_workspace_size(ctypes.byref(shape), sparse_block_size, sparse_mode, int(deterministic),
                                        ctypes.byref(n)))
    return n.value


def sfa_grad(query, key, value, sparse_indices, d_out, out, softmax_max, softmax_sum, query_rope, key_rope, *,
             scale: float, sparse_block_size: int, layout: str, sparse_mode: int, deterministic: bool = False,
             actual_seq_lengths_q=None, actual_seq_lengths_kv=None, pre_tokens: int = 2 ** 31 - 1,
             next_tokens: int = 2 ** 31 - 1, workspace: Optional[torch.Tensor] = None, outputs=None, stream=None):
    """Backward of top-k sparse attention; returns (dQuery, dKey, dValue, dQueryRope, dKeyRope)."""
    lib = N.load()
    dt = query.dtype
    for name, t in (("query", query), ("key", key), ("value", value), ("d_out", d_out), ("out", out),
                    ("query_rope", query_rope), ("key_rope", key_rope)):
        _check16(name, t, dt)
    shape = sfa_shape(query, key, query_rope, sparse_indices, layout, actual_seq_lengths_q)
    _check_sfa_inputs(shape, query, key, value, sparse_indices, query_rope, key_rope, d_out, out, softmax_max,
                      softmax_sum)
    _check_cuda(_sfa_named(query, key, value, sparse_indices, query_rope, key_rope, d_out, out, softmax_max,
                           softmax_sum))
    sq = _seqlens(actual_seq_lengths_q, layout, shape.B)
    skv = _seqlens(actual_seq_lengths_kv, layout, shape.B)
    ws_bytes = sfa_grad_workspace_size(shape, sparse_block_size, sparse_mode, deterministic)
    workspace = _workspace(workspace, ws_bytes, query.device)
    if outputs is None:
        outputs = (torch.empty_like(query), torch.empty_like(key), torch.empty_like(key),
                   torch.empty_like(query_rope), torch.empty_like(key_rope))
    dq, dk, dv, dqr, dkr = outputs
    _check_outputs((("d_query", dq), ("d_key", dk), ("d_value", dv), ("d_query_rope", dqr), ("d_key_rope", dkr)),
                   ((dt, query.numel()), (dt, key.numel()), (dt, key.numel()), (dt, query_rope.numel()),
                    (dt, key_rope.numel())))
    N.check(lib.sfa_grad(_p(query), _p(key), _p(value), _p(sparse_indices), _p(d_out), _p(out), _p(softmax_max),
                         _p(softmax_sum), _p(sq), _p(skv), _p(query_rope), _p(key_rope), float(scale),
                         int(sparse_block_size), int(sparse_mode), int(pre_tokens), int(next_tokens),
                         int(deterministic), ctypes.byref(shape), _p(workspace), workspace.numel(), _stream(stream),
                         _p(dq), _p(dk), _p(dv), _p(dqr), _p(dkr)))
    return dq, dk, dv, dqr, dkr


def sfa_dkv_accumulator(query, key, query_rope, sparse_indices, *, layout: str, deterministic: bool,
                        actual_seq_lengths_q=None):
    """Zeroed key-side accumulator for sfa_grad_rows: [T2, 1088] (dKey | dKeyRope | dValue), fp32,
    or int64 fixed point when deterministic."""
    lib = N.load()
    shape = sfa_shape(query, key, query_rope, sparse_indices, layout, actual_seq_lengths_q)
    n = ctypes.c_size_t()
    N.check(lib.sfa_dkv_accum_size(ctypes.byref(shape), int(deterministic), ctypes.byref(n)))
    dt = torch.int64 if deterministic else torch.float32
    return torch.zeros(shape.T2, n.value // (shape.T2 * (8 if deterministic else 4)), dtype=dt, device=query.device)


def _check_accum(dkv_accum, shape, deterministic):
    _need(dkv_accum.is_contiguous() and dkv_accum.dtype == (torch.int64 if deterministic else torch.float32),
          "dkv_accum: contiguous, int64 when deterministic else float32")
    _need(dkv_accum.numel() == shape.T2 * ACC_WIDTH, f"dkv_accum: {dkv_accum.numel()} elements, expected "
          f"{shape.T2 * ACC_WIDTH}")


def _check_absmax(dout_absmax, deterministic):
    if deterministic:
        _need(dout_absmax is not None, "deterministic: dout_absmax (from dout_absmax()) is required")
    if dout_absmax is not None:
        _need(dout_absmax.dtype == torch.float32 and dout_absmax.numel() == 1, "dout_absmax: one fp32 element")


def dout_absmax(d_out, query, key, query_rope, sparse_indices, *, layout: str, row_begin: int = 0,
                row_end: Optional[int] = None, actual_seq_lengths_q=None, into: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    """max|d_out| over query rows [row_begin, row_end), max-merged into `into` (a 1-element fp32 CUDA
    tensor, zeroed here when not given).  It sets the fixed-point grid of deterministic row ranges."""
    lib = N.load()
    shape = sfa_shape(query, key, query_rope, sparse_indices, layout, actual_seq_lengths_q)
    _check16("d_out", d_out, query.dtype)
    _check_numel((("d_out", d_out, shape.T1 * shape.N1 * shape.D),))
    _check_cuda((("d_out", d_out),))
    if into is None:
        into = torch.zeros(1, dtype=torch.float32, device=d_out.device)
    _check_absmax(into, False)
    _check_cuda((("into", into),))
    N.check(lib.sfa_dout_absmax(_p(d_out), ctypes.byref(shape), int(row_begin),
                                int(shape.T1 if row_end is None else row_end), _stream(stream), _p(into)))
    return into


def sfa_grad_rows(query, key, value, sparse_indices, d_out, out, softmax_max, softmax_sum, query_rope, key_rope, *,
                  row_begin: int, row_end: int, dkv_accum: torch.Tensor, scale: float, sparse_block_size: int,
                  layout: str, sparse_mode: int, deterministic: bool = False, dout_absmax=None,
                  actual_seq_lengths_q=None, actual_seq_lengths_kv=None, workspace: Optional[torch.Tensor] = None,
                  d_query=None, d_query_rope=None, stream=None):
    """Backward of query rows [row_begin, row_end) (flattened row index): writes those rows of
    (dQuery, dQueryRope) and adds their dKey / dKeyRope / dValue contributions into `dkv_accum`
    (from sfa_dkv_accumulator).  Deterministic mode needs `dout_absmax`: max|d_out| over every row
    that goes into the accumulator (see dout_absmax()).  Returns (dQuery, dQueryRope)."""
    lib = N.load()
    dt = query.dtype
    for name, t in (("query", query), ("key", key), ("value", value), ("d_out", d_out), ("out", out),
                    ("query_rope", query_rope), ("key_rope", key_rope)):
        _check16(name, t, dt)
    shape = sfa_shape(query, key, query_rope, sparse_indices, layout, actual_seq_lengths_q)
    _check_sfa_inputs(shape, query, key, value, sparse_indices, query_rope, key_rope, d_out, out, softmax_max,
                      softmax_sum)
    _check_accum(dkv_accum, shape, deterministic)
    _check_absmax(dout_absmax, deterministic)
    _check_cuda(_sfa_named(query, key, value, sparse_indices, query_rope, key_rope, d_out, out, softmax_max,
                           softmax_sum) + (("dkv_accum", dkv_accum), ("dout_absmax", dout_absmax)))
    sq = _seqlens(actual_seq_lengths_q, layout, shape.B)
    skv = _seqlens(actual_seq_lengths_kv, layout, shape.B)
    ws_bytes = sfa_grad_workspace_size(shape, sparse_block_size, sparse_mode, deterministic)
    workspace = _workspace(workspace, ws_bytes, query.device)
    if d_query is None:
        d_query = torch.zeros_like(query)
    if d_query_rope is None:
        d_query_rope = torch.zeros_like(query_rope)
    _check_outputs((("d_query", d_query), ("d_query_rope", d_query_rope)),
                   ((dt, query.numel()), (dt, query_rope.numel())))
    N.check(lib.sfa_grad_rows(_p(query), _p(key), _p(value), _p(sparse_indices), _p(d_out), _p(out),
                              _p(softmax_max), _p(softmax_sum), _p(sq), _p(skv), _p(query_rope), _p(key_rope),
                              float(scale), int(sparse_block_size), int(sparse_mode), int(deterministic),
                              int(row_begin), int(row_end), ctypes.byref(shape), _p(workspace), workspace.numel(),
                              _stream(stream), _p(dkv_accum), _p(dout_absmax), _p(d_query), _p(d_query_rope)))
    return d_query, d_query_rope


def sfa_dkv_finalize(dkv_accum, query, key, query_rope, sparse_indices, *, layout: str, deterministic: bool,
                     dout_absmax=None, scale: float = 1.0, actual_seq_lengths_q=None, outputs=None, stream=None):
    """Casts a (summed) key-side accumulator into 16-bit (dKey, dValue, dKeyRope).  Deterministic mode
    needs the `dout_absmax` and `scale` the accumulator was filled with."""
    lib = N.load()
    shape = sfa_shape(query, key, query_rope, sparse_indices, layout, actual_seq_lengths_q)
    _check_accum(dkv_accum, shape, deterministic)
    _check_absmax(dout_absmax, deterministic)
    _check_cuda((("dkv_accum", dkv_accum), ("dout_absmax", dout_absmax)))
    kr_shape = key.shape[:-1] + (query_rope.shape[-1],)
    if outputs is None:
        outputs = (torch.empty_like(key), torch.empty_like(key),
                   torch.empty(kr_shape, dtype=key.dtype, device=key.device))
    dk, dv, dkr = outputs
    n_kr = shape.T2 * shape.N2 * shape.Dr
    _check_outputs((("d_key", dk), ("d_value", dv), ("d_key_rope", dkr)),
                   ((key.dtype, key.numel()), (key.dtype, key.numel()), (key.dtype, n_kr)))
    N.check(lib.sfa_dkv_finalize(_p(dkv_accum), ctypes.byref(shape), int(deterministic), _p(dout_absmax),
                                 float(scale), _stream(stream), _p(dk), _p(dv), _p(dkr)))
    return dk, dv, dkr


def sfa_fwd(query, key, value, sparse_indices, query_rope, key_rope, *, scale: float, sparse_block_size: int,
            layout: str, sparse_mode: int, actual_seq_lengths_q=None, actual_seq_lengths_kv=None, workspace=None,
            stream=None):
    """Forward of top-k sparse attention; returns (out, softmaxMax, softmaxSum)."""
    lib = N.load()
    dt = query.dtype
    for name, t in (("query", query), ("key", key), ("value", value), ("query_rope", query_rope),
                    ("key_rope", key_rope)):
        _check16(name, t, dt)
    shape = sfa_shape(query, key, query_rope, sparse_indices, layout, actual_seq_lengths_q)
    _check_sfa_inputs(shape, query, key, value, sparse_indices, query_rope, key_rope)
    _check_cuda(_sfa_named(query, key, value, sparse_indices, query_rope, key_rope))
    sq = _seqlens(actual_seq_lengths_q, layout, shape.B)
    skv = _seqlens(actual_seq_lengths_kv, layout, shape.B)
    n = ctypes.c_size_t()
    N.check(lib.sfa_fwd_workspace_size(ctypes.byref(shape), sparse_block_size, sparse_mode, ctypes.byref(n)))
    ws = _workspace(workspace, n.value, query.device)
    out = torch.empty_like(query)
    stat_shape = query.shape[:-1]
    smax = torch.empty(stat_shape, dtype=torch.float32, device=query.device)
    ssum = torch.empty(stat_shape, dtype=torch.float32, device=query.device)
    N.check(lib.sfa_fwd(_p(query), _p(key), _p(value), _p(sparse_indices), _p(sq), _p(skv), _p(query_rope),
                        _p(key_rope), float(scale), int(sparse_block_size), int(sparse_mode), ctypes.byref(shape),
                        _p(ws), ws.numel(), _stream(stream), _p(out), _p(smax), _p(ssum)))
    return out, smax, ssum


def compact_indices(sparse_indices, key, query, query_rope, *, sparse_block_size: int, layout: str,
                    sparse_mode: int, actual_seq_lengths_q=None, actual_seq_lengths_kv=None, stream=None):
    """Index compaction step; returns (blocks [T1, topk], nblocks [T1], nrows [T1]) int32."""
    lib = N.load()
    shape = sfa_shape(query, key, query_rope, sparse_indices, layout, actual_seq_lengths_q)
    _need(sparse_indices.dtype == torch.int32 and sparse_indices.is_contiguous(),
          "sparse_indices: int32 contiguous tensor")
    _check_numel((("sparse_indices", sparse_indices, shape.T1 * shape.N2 * shape.topk),))
    _check_cuda((("sparse_indices", sparse_indices),))
    sq = _seqlens(actual_seq_lengths_q, layout, shape.B)
    skv = _seqlens(actual_seq_lengths_kv, layout, shape.B)
    dev = sparse_indices.device
    blocks = torch.full((shape.T1, shape.topk), -7, dtype=torch.int32, device=dev)
    nb = torch.empty(shape.T1, dtype=torch.int32, device=dev)
    nr = torch.empty(shape.T1, dtype=torch.int32, device=dev)
    N.check(lib.sfa_compact_indices(_p(sparse_indices), _p(sq), _p(skv), int(sparse_block_size), int(sparse_mode),
                                    ctypes.byref(shape), _stream(stream), _p(blocks), _p(nb), _p(nr)))
    return blocks, nb, nr


def key_rows(sparse_indices, key, query, query_rope, *, sparse_block_size: int, layout: str, sparse_mode: int,
             sorted_blocks: bool = False, block_aligned: bool = False, actual_seq_lengths_q=None,
             actual_seq_lengths_kv=None, stream=None):
    """Gathered key rows per query row (sfa_key_rows); returns (blocks [T1, topk], nblocks [T1],
    rows [T1, topk*bs], count [T1]) int32.  Block-aligned lists flag padding slots with bit 31."""
    lib = N.load()
    shape = sfa_shape(query, key, query_rope, sparse_indices, layout, actual_seq_lengths_q)
    _need(sparse_indices.dtype == torch.int32 and sparse_indices.is_contiguous(),
          "sparse_indices: int32 contiguous tensor")
    _check_numel((("sparse_indices", sparse_indices, shape.T1 * shape.N2 * shape.topk),))
    _check_cuda((("sparse_indices", sparse_indices),))
    sq = _seqlens(actual_seq_lengths_q, layout, shape.B)
    skv = _seqlens(actual_seq_lengths_kv, layout, shape.B)
    dev = sparse_indices.device
    blocks = torch.full((shape.T1, shape.topk), -7, dtype=torch.int32, device=dev)
    nb = torch.empty(shape.T1, dtype=torch.int32, device=dev)
    rows = torch.full((shape.T1, shape.topk * sparse_block_size), -7, dtype=torch.int32, device=dev)
    cnt = torch.empty(shape.T1, dtype=torch.int32, device=dev)
    N.check(lib.sfa_key_rows(_p(sparse_indices), _p(sq), _p(skv), int(sparse_block_size), int(sparse_mode),
                             ctypes.byref(shape), int(sorted_blocks), int(block_aligned), _stream(stream), _p(blocks),
                             _p(nb), _p(rows), _p(cnt)))
    return blocks, nb, rows, cnt


def softmax_grad_rowsum(d_out, out, key, query_rope, sparse_indices, *, layout: str, actual_seq_lengths_q=None,
                        stream=None):
    """FlashSoftmaxGrad(dO, O): fp32 [T1, N1] row sums of dO o O."""
    lib = N.load()
    shape = sfa_shape(d_out, key, query_rope, sparse_indices, layout, actual_seq_lengths_q)
    _check16("d_out", d_out, d_out.dtype)
    _check16("out", out, d_out.dtype)
    _check_numel((("out", out, d_out.numel()),))
    _check_cuda((("d_out", d_out), ("out", out)))
    res = torch.empty(shape.T1 * shape.N1, dtype=torch.float32, device=d_out.device)
    N.check(lib.sfa_softmax_grad_rowsum(_p(d_out), _p(out), ctypes.byref(shape), _stream(stream), _p(res)))
    return res.view(shape.T1, shape.N1)


def _fa_shape(q, k, cu_q, cu_kv) -> N.FaShape:
    s = N.FaShape()
    _need(q.dtype in _DT, "q must be bf16 or fp16")
    _need(q.dim() == 3 and k.dim() == 3, "TND tensors are 3-D")
    _need(len(cu_q) == len(cu_kv), "cu_seqlens_q and cu_seqlens_kv need the same length B")
    s.dtype = _DT[q.dtype]
    s.B = len(cu_q)
    s.T1, s.Nq, s.D = q.shape
    s.T2, s.Nkv, _ = k.shape
    return s


def _check_fa_inputs(s, q, k=None, v=None, dy=None, softmax_max=None, softmax_sum=None, attention_in=None):
    for name, t in (("softmax_max", softmax_max), ("softmax_sum", softmax_sum)):
        if t is not None:
            _check_f32(name, t)
    _check_numel((("k", k, s.T2 * s.Nkv * s.D), ("v", v, s.T2 * s.Nkv * s.D), ("dy", dy, s.T1 * s.Nq * s.D),
                  ("attention_in", attention_in, s.T1 * s.Nq * s.D), ("softmax_max", softmax_max, s.T1 * s.Nq * 8),
                  ("softmax_sum", softmax_sum, s.T1 * s.Nq * 8)))
    _check_cuda((("q", q), ("k", k), ("v", v), ("dy", dy), ("attention_in", attention_in),
                 ("softmax_max", softmax_max), ("softmax_sum", softmax_sum)))


def _host_i64(x: Sequence[int]):
    a = np.ascontiguousarray(np.asarray(x, dtype=np.int64))
    return a, a.ctypes.data_as(ctypes.c_void_p)


def fa_grad(q, k, v, dy, softmax_max, softmax_sum, attention_in, cu_seqlens_q, cu_seqlens_kv, *, scale: float,
            sparse_mode: int, deterministic: bool = False, keep_prob: float = 1.0, pre_tokens: int = 65536,
            next_tokens: int = 65536, workspace=None, outputs=None, stream=None):
    """Dense varlen FA backward (TND); cu_seqlens_* are host cumulative end offsets. Returns (dq, dk, dv)."""
    lib = N.load()
    for name, t in (("q", q), ("k", k), ("v", v), ("dy", dy), ("attention_in", attention_in)):
        _check16(name, t, q.dtype)
    shape = _fa_shape(q, k, cu_seqlens_q, cu_seqlens_kv)
    _check_fa_inputs(shape, q, k, v, dy, softmax_max, softmax_sum, attention_in)
    n = ctypes.c_size_t()
    N.check(lib.fa_grad_workspace_size(ctypes.byref(shape), int(sparse_mode), int(deterministic), ctypes.byref(n)))
    workspace = _workspace(workspace, n.value, q.device)
    if outputs is None:
        outputs = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    dq, dk, dv = outputs
    _check_outputs((("dq", dq), ("dk", dk), ("dv", dv)),
                   ((q.dtype, q.numel()), (q.dtype, k.numel()), (q.dtype, v.numel())))
    aq, pq = _host_i64(cu_seqlens_q)
    akv, pkv = _host_i64(cu_seqlens_kv)
    N.check(lib.fa_grad(_p(q), _p(k), _p(v), _p(dy), _p(softmax_max), _p(softmax_sum), _p(attention_in), pq, pkv,
                        float(scale), float(keep_prob), int(pre_tokens), int(next_tokens), int(shape.Nq),
                        int(sparse_mode), int(deterministic), ctypes.byref(shape), _p(workspace), workspace.numel(),
                        _stream(stream), _p(dq), _p(dk), _p(dv)))
    del aq, akv
    return dq, dk, dv


def fa_fwd(q, k, v, cu_seqlens_q, cu_seqlens_kv, *, scale: float, sparse_mode: int, stream=None):
    """Dense varlen FA forward (TND). Returns (out, softmaxMax [T1,Nq,8], softmaxSum [T1,Nq,8])."""
    lib = N.load()
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check16(name, t, q.dtype)
    shape = _fa_shape(q, k, cu_seqlens_q, cu_seqlens_kv)
    _check_fa_inputs(shape, q, k, v)
    n = ctypes.c_size_t()
    N.check(lib.fa_fwd_workspace_size(ctypes.byref(shape), int(sparse_mode), ctypes.byref(n)))
    ws = torch.empty(max(n.value, 1), dtype=torch.uint8, device=q.device)
    out = torch.empty_like(q)
    smax = torch.empty(q.shape[0], q.shape[1], 8, dtype=torch.float32, device=q.device)
    ssum = torch.empty_like(smax)
    aq, pq = _host_i64(cu_seqlens_q)
    akv, pkv = _host_i64(cu_seqlens_kv)
    N.check(lib.fa_fwd(_p(q), _p(k), _p(v), pq, pkv, float(scale), int(sparse_mode), ctypes.byref(shape), _p(ws),
                       ws.numel(), _stream(stream), _p(out), _p(smax), _p(ssum)))
    del aq, akv
    return out, smax, ssum


def lig_shape(query: torch.Tensor, key: torch.Tensor, query_index: torch.Tensor, key_index: torch.Tensor,
              layout: str, actual_seq_lengths_query=None, query_rope: Optional[torch.Tensor] = None) -> N.LigShape:
    """Sizes of a dense lightning-indexer gradient call from its tensors (Dr from query_rope,
    64 when it is not given)."""
    s = N.LigShape()
    _need(query.dtype in _DT, "query must be bf16 or fp16")
    s.dtype = _DT[query.dtype]
    if layout == "BSND":
        _need(query.dim() == 4 and key.dim() == 4, "BSND tensors are 4-D")
        s.layout = N.LAYOUT_BSND
        s.B, s.S1, s.N1, s.D = query.shape
        _, s.S2, _, _ = key.shape
        s.T1, s.T2 = s.B * s.S1, s.B * s.S2
        _, _, s.G, s.Di = query_index.shape
    elif layout == "TND":
        _need(query.dim() == 3 and key.dim() == 3, "TND tensors are 3-D")
        s.layout = N.LAYOUT_TND
        s.T1, s.N1, s.D = query.shape
        s.T2 = key.shape[0]
        s.S1 = s.S2 = 0
        _need(actual_seq_lengths_query is not None, "TND needs actual sequence lengths")
        s.B = actual_seq_lengths_query.numel()
        _, s.G, s.Di = query_index.shape
    else:
        raise ValueError(f"layout {layout!r}")
    s.Dr = 64 if query_rope is None else query_rope.shape[-1]
    return s


def lig_kl_grad_workspace_size(shape: N.LigShape, sparse_mode: int) -> int:
    n = ctypes.c_size_t()
    N.check(N.load().lig_kl_grad_workspace_size(ctypes.byref(shape), int(sparse_mode), ctypes.byref(n)))
    return n.value


def lig_kl_grad(query, key, query_index, key_index, weights, softmax_max, softmax_sum, softmax_max_index,
                softmax_sum_index, query_rope, key_rope, *, scale: float, layout: str, sparse_mode: int,
                actual_seq_lengths_query=None, actual_seq_lengths_key=None, pre_tokens: int = 65536,
                next_tokens: int = 65536, workspace=None, outputs=None, stream=None):
    """Dense lightning-indexer gradient with KL loss (lig_kl_grad in include/sfa.h).
    Returns (dQueryIndex, dKeyIndex, dWeights, loss) with loss a 1-element fp32 CUDA tensor."""
    lib = N.load()
    for name, t in (("query", query), ("key", key), ("query_index", query_index), ("key_index", key_index),
                    ("weights", weights), ("query_rope", query_rope), ("key_rope", key_rope)):
        _check16(name, t, query.dtype)
    for name, t in (("softmax_max", softmax_max), ("softmax_sum", softmax_sum),
                    ("softmax_max_index", softmax_max_index), ("softmax_sum_index", softmax_sum_index)):
        _check_f32(name, t)
    for name, t in (("actual_seq_lengths_query", actual_seq_lengths_query),
                    ("actual_seq_lengths_key", actual_seq_lengths_key)):
        _need(t is None or (t.dtype == torch.int64 and t.is_contiguous()), f"{name}: int64 tensor")
    if layout == "TND":
        _need(actual_seq_lengths_key is not None, "TND needs actual_seq_lengths_key")
    shape = lig_shape(query, key, query_index, key_index, layout, actual_seq_lengths_query, query_rope)
    # the library sees raw pointers: every tensor must hold exactly the elements its layout implies
    T1, T2 = shape.T1, shape.T2
    for name, t in (("actual_seq_lengths_query", actual_seq_lengths_query),
                    ("actual_seq_lengths_key", actual_seq_lengths_key)):
        _need(t is None or t.numel() == shape.B, f"{name}: {shape.B} elements expected")
    for name, t, n in (("query_index", query_index, T1 * shape.G * shape.Di),
                       ("key", key, T2 * shape.D), ("key_index", key_index, T2 * shape.Di),
                       ("weights", weights, T1 * shape.G), ("query_rope", query_rope, T1 * shape.N1 * shape.Dr),
                       ("key_rope", key_rope, T2 * shape.Dr), ("softmax_max", softmax_max, T1 * shape.N1),
                       ("softmax_sum", softmax_sum, T1 * shape.N1), ("softmax_max_index", softmax_max_index, T1),
                       ("softmax_sum_index", softmax_sum_index, T1)):
        _need(t.numel() == n, f"{name}: {t.numel()} elements, expected {n}")
    _check_cuda((("query", query), ("key", key), ("query_index", query_index), ("key_index", key_index),
                 ("weights", weights), ("query_rope", query_rope), ("key_rope", key_rope),
                 ("softmax_max", softmax_max), ("softmax_sum", softmax_sum),
                 ("softmax_max_index", softmax_max_index), ("softmax_sum_index", softmax_sum_index),
                 ("actual_seq_lengths_query", actual_seq_lengths_query),
                 ("actual_seq_lengths_key", actual_seq_lengths_key)))
    need = lig_kl_grad_workspace_size(shape, sparse_mode)
    workspace = _workspace(workspace, need, query.device)
    if outputs is None:
        outputs = (torch.empty_like(query_index), torch.empty_like(key_index), torch.empty_like(weights),
                   torch.empty(1, dtype=torch.float32, device=query.device))
    dqi, dki, dw, loss = outputs
    dt = query.dtype
    _check_outputs((("d_query_index", dqi), ("d_key_index", dki), ("d_weights", dw), ("loss", loss)),
                   ((dt, T1 * shape.G * shape.Di), (dt, T2 * shape.Di), (dt, T1 * shape.G), (torch.float32, 1)))
    N.check(lib.lig_kl_grad(_p(query), _p(key), _p(query_index), _p(key_index), _p(weights), _p(softmax_max),
                            _p(softmax_sum), _p(softmax_max_index), _p(softmax_sum_index), _p(query_rope),
                            _p(key_rope), _p(actual_seq_lengths_query), _p(actual_seq_lengths_key), float(scale),
                            int(sparse_mode), int(pre_tokens), int(next_tokens), ctypes.byref(shape), _p(workspace),
                            workspace.numel(), _stream(stream), _p(dqi), _p(dki), _p(dw), _p(loss)))
    return dqi, dki, dw, loss


def workspace_status(workspace: torch.Tensor, stream=None) -> int:
    """Waits for `stream` and returns the wait-site code the last call left in the workspace's
    error word: 0 when every device-side wait was satisfied, else the site that gave up."""
    lib = N.load()
    site = ctypes.c_int32(0)
    st = lib.sfa_workspace_status(_p(workspace), _stream(stream), ctypes.byref(site))
    if st not in (N.SFA_OK, N.SFA_ERR_TIMEOUT):
        N.check(st)
    return int(site.value)


def set_wait_limit(limit_ns: int) -> None:
    """Limit of every device-side wait of the fused kernels launched afterwards from this
    thread (0: the default 4 s)."""
    N.check(N.load().sfa_set_wait_limit(int(limit_ns)))
