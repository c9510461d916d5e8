"""Plain CPU oracle for top-k sparse attention (forward + backward) and the dense
varlen FlashAttention backward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or run
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline``
/ ``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the
CUDA library (no kernels, headers, tables or helpers); both sides only consume
the same seeded inputs from ``workloads``.

Everything is numpy in float64 (``dtype`` may be lowered to float32 for the
bounded CPU-baseline timing runs).  Each function follows the definition on
the source pages, written out without blocking, fusion or reordering:

* SparseFlashAttentionGrad (gitcode ops-transformer README, "attention/
  sparse_flash_attention_grad"), section 功能说明 (function description): the
  Gather of key/value by topkIndices in blocks of selectedBlockSize, then
  stage 1 (dP = dO.V^T, dV = P^T.dO), stage 2 (dS = P o (dP - FlashSoftmaxGrad(dO, O)))
  and stage 3 (dQ = dS.K/sqrt(d), dK = dS^T.Q/sqrt(d)); 参数说明 (parameters) for
  the MLA rope split and the outputs; 约束说明 (constraints) for sparseMode 0/3.
* aclnnFlashAttentionUnpaddingScoreGrad (coreui.cn "CANN算子库FlashAttention反向
  梯度计算"), section 计算公式 (formula): S, P, Y of the forward and dV = P^T.dY,
  dQ = dS.K/sqrt(d), dK = dS^T.Q/sqrt(d); 约束说明 for TND, GQA (Nq/Nkv integer)
  and the [T, N, 8] softmaxMax/softmaxSum layout.

Readings taken where the pages are silent or garbled (each is listed in the
repository's design notes):

* stage 2's "@" is the elementwise product, FlashSoftmaxGrad(dO, O) is the row
  sum over the value dims of dO o O, broadcast over keys;
* the 1/sqrt(d) of stage 3 is the scaleValue attribute, used in S, dQ and dK;
* softmaxMax / softmaxSum are the max of the *scaled* scores and the sum of
  exp(scaled - max); they are used as given, never recomputed;
* an index i selects rows [i*bs, i*bs+bs) of its own batch/sequence; negative
  indices and blocks starting at or past S2_b are skipped; rows past S2_b or
  past the sparseMode-3 causal bound are dropped one by one; duplicates count
  with multiplicity;
* sparseMode 3 keeps key j for query position i iff j <= i + S2_b - S1_b;
* a row with no valid key has O = 0, softmaxMax = 0, softmaxSum = 0, and a
  softmaxSum of 0 gives P = 0;
* dKey excludes dValue's share even though value aliases key.

Parity status: every public function is pinned by ``tests/test_oracle_pins.py``
(finite differences, a torch SDPA special case, invariants, hand-worked index
cases and the page-2 all-ones worked example).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional, Sequence

import numpy as np

LAYOUT_BSND = "BSND"
LAYOUT_TND = "TND"


# ----------------------------------------------------------------------------
# Batch / sequence bookkeeping
# ----------------------------------------------------------------------------
@dataclass(frozen=True)
class Span:
    """One batch (BSND) or one packed sequence (TND)."""

    q_start: int  # first query row of this batch in the flattened [T1, ...] view
    q_len: int  # S1_b: valid query tokens
    kv_start: int  # first key row of this batch in the flattened [T2, ...] view
    kv_len: int  # S2_b: valid key tokens


def make_spans(layout: str, B: int, S1: int, S2: int,
               seqlens_q: Optional[Sequence[int]], seqlens_kv: Optional[Sequence[int]]) -> List[Span]:
    """Per-batch spans.

    BSND (SparseFlashAttentionGrad, 参数说明: actualSeqLengthsQuery/kv are "the
    valid token count of each batch"): rows are padded to S1/S2 per batch;
    ``seqlens_*`` are per-batch lengths, ``None`` meaning the full S1/S2.
    TND (aclnnFlashAttentionUnpaddingScoreGrad, 约束说明: T is B and S packed
    tightly): ``seqlens_*`` are cumulative end offsets, length B, last = T.
    """
    spans = []
    if layout == LAYOUT_BSND:
        for b in range(B):
            lq = S1 if seqlens_q is None else int(seqlens_q[b])
            lk = S2 if seqlens_kv is None else int(seqlens_kv[b])
            spans.append(Span(b * S1, lq, b * S2, lk))
    elif layout == LAYOUT_TND:
        pq = pk = 0
        for b in range(B):
            eq, ek = int(seqlens_q[b]), int(seqlens_kv[b])
            spans.append(Span(pq, eq - pq, pk, ek - pk))
            pq, pk = eq, ek
    else:
        raise ValueError(layout)
    return spans


def selected_rows(idx_row: np.ndarray, block_size: int, q_pos: int, q_len: int, kv_len: int,
                  sparse_mode: int) -> List[int]:
    """Key rows (local to the batch) that one query token attends to.

    Gather of key/value by topkIndices[i] in blocks of selectedBlockSize
    (SparseFlashAttentionGrad, 功能说明), in index order, with multiplicity.
    sparseMode 3 is the lower triangle split at the right vertex (约束说明):
    key j is kept for query position q_pos iff j <= q_pos + kv_len - q_len.
    """
    rows: List[int] = []
    for i in idx_row.tolist():
        if i < 0:
            continue
        start = i * block_size
        if start >= kv_len:
            continue
        for j in range(start, start + block_size):
            if j >= kv_len:
                break
            if sparse_mode == 3 and j > q_pos + kv_len - q_len:
                continue
            rows.append(j)
    return rows


# ----------------------------------------------------------------------------
# Sparse attention (MLA shape: D latent + Dr rope, N2 = 1)
# ----------------------------------------------------------------------------
def _as(x, dtype):
    return np.asarray(x, dtype=dtype)


def _row(x, t, dtype):
    return np.asarray(x[t], dtype=dtype)


def sfa_forward(q, k, v, indices, q_rope, k_rope, scale: float, block_size: int, sparse_mode: int,
                layout: str, B: int, S1: int, S2: int,
                seqlens_q=None, seqlens_kv=None, dtype=np.float64, tokens=None):
    """O, softmaxMax, softmaxSum of top-k sparse attention.

    q: [T1, N1, D], k/v: [T2, D] (N2 = 1 squeezed), q_rope: [T1, N1, Dr],
    k_rope: [T2, Dr], indices: [T1, topk] (N2 squeezed); BSND tensors are passed
    flattened to T1 = B*S1 / T2 = B*S2 rows.  Query-side arguments only need
    ``len()`` and row indexing, and are converted one row at a time.
    Forward of the attention structure (aclnnFlashAttentionUnpaddingScoreGrad,
    计算公式: S = QK^T*scale, P = Softmax(S), Y = PV) restricted to the gathered
    rows.  ``tokens`` restricts the work to a subset of flattened query rows; the
    outputs then hold only those rows, in ascending row order.
    Returns out [T1, N1, Dv], softmax_max [T1, N1], softmax_sum [T1, N1].
    """
    k, v, k_rope = (_as(a, dtype) for a in (k, v, k_rope))
    T1 = len(q)
    sel = list(range(T1)) if tokens is None else sorted(int(t) for t in tokens)
    N1 = _row(q, sel[0] if sel else 0, dtype).shape[0]
    Dv = v.shape[1]
    where = {t: i for i, t in enumerate(sel)}
    out = np.zeros((len(sel), N1, Dv), dtype)
    smax = np.zeros((len(sel), N1), dtype)
    ssum = np.zeros((len(sel), N1), dtype)
    kt_all = np.concatenate([k, k_rope], axis=1)
    for sp in make_spans(layout, B, S1, S2, seqlens_q, seqlens_kv):
        for pos in range(sp.q_len):
            t = sp.q_start + pos
            if t not in where:
                continue
            rows = selected_rows(np.asarray(indices[t]), block_size, pos, sp.q_len, sp.kv_len, sparse_mode)
            if not rows:
                continue
            i = where[t]
            g = sp.kv_start + np.asarray(rows)
            qt = np.concatenate([_row(q, t, dtype), _row(q_rope, t, dtype)], axis=1)
            s = scale * (qt @ kt_all[g].T)  # [N1, n]
            m = s.max(axis=1)
            e = np.exp(s - m[:, None])
            l = e.sum(axis=1)
            out[i] = (e / l[:, None]) @ v[g]
            smax[i] = m
            ssum[i] = l
    return out, smax, ssum


def sfa_backward(q, k, v, indices, d_out, out, softmax_max, softmax_sum, q_rope, k_rope,
                 scale: float, block_size: int, sparse_mode: int, layout: str, B: int, S1: int, S2: int,
                 seqlens_q=None, seqlens_kv=None, dtype=np.float64, tokens=None, return_ds: bool = False):
    """dQuery, dKey, dValue, dQueryRope, dKeyRope of top-k sparse attention.

    Per query token t, with J_t the gathered rows (SparseFlashAttentionGrad,
    功能说明 Gather) and Q~ = [q || q_rope], K~ = [k || k_rope] (参数说明, MLA rope):
      P  = exp(scale*Q~.K~^T - softmaxMax) / softmaxSum          (stats as given)
      dP = dO.V^T ;  dV[J_t] += P^T.dO                            (stage 1)
      dS = P o (dP - rowsum(dO o O))                              (stage 2)
      dQ~ = scale*dS.K~ ;  dK~[J_t] += scale*dS^T.Q~              (stage 3)
    Scatter-adds go through ``np.add.at`` so repeated rows accumulate.
    Query-side arguments only need ``len()`` and row indexing.  ``tokens``
    restricts the sums to a subset of query rows (sub-problem checks); dQuery /
    dQueryRope then hold only those rows, in ascending row order.
    """
    k, v, k_rope = (_as(a, dtype) for a in (k, v, k_rope))
    T1 = len(q)
    sel = list(range(T1)) if tokens is None else sorted(int(t) for t in tokens)
    N1, D = _row(q, sel[0] if sel else 0, dtype).shape
    Dr = _row(q_rope, sel[0] if sel else 0, dtype).shape[1]
    T2 = k.shape[0]
    where = {t: i for i, t in enumerate(sel)}
    kt_all = np.concatenate([k, k_rope], axis=1)
    dqt = np.zeros((len(sel), N1, D + Dr), dtype)
    dkt = np.zeros((T2, D + Dr), dtype)
    dv = np.zeros_like(v)
    ds_rows = {}
    for sp in make_spans(layout, B, S1, S2, seqlens_q, seqlens_kv):
        for pos in range(sp.q_len):
            t = sp.q_start + pos
            if t not in where:
                continue
            rows = selected_rows(np.asarray(indices[t]), block_size, pos, sp.q_len, sp.kv_len, sparse_mode)
            if not rows:
                continue
            g = sp.kv_start + np.asarray(rows)
            qt = np.concatenate([_row(q, t, dtype), _row(q_rope, t, dtype)], axis=1)  # [N1, D+Dr]
            do = _row(d_out, t, dtype)
            kt = kt_all[g]  # [n, D+Dr]
            vt = v[g]  # [n, Dv]
            s = scale * (qt @ kt.T)  # [N1, n]
            l = _row(softmax_sum, t, dtype)
            inv_l = np.where(l == 0, 0.0, 1.0 / np.where(l == 0, 1.0, l))
            p = np.exp(s - _row(softmax_max, t, dtype)[:, None]) * inv_l[:, None]
            dp = do @ vt.T  # stage 1
            np.add.at(dv, g, p.T @ do)  # stage 1
            dsum = (do * _row(out, t, dtype)).sum(axis=1)  # FlashSoftmaxGrad(dO, O)
            ds = p * (dp - dsum[:, None])  # stage 2
            dqt[where[t]] = scale * (ds @ kt)  # stage 3
            np.add.at(dkt, g, scale * (ds.T @ qt))  # stage 3
            if return_ds:
                ds_rows[t] = ds
    res = (dqt[:, :, :D], dkt[:, :D], dv, dqt[:, :, D:], dkt[:, D:])
    if return_ds:
        return res + (ds_rows,)
    return res


# ----------------------------------------------------------------------------
# Dense varlen FlashAttention (TND, GQA, sparseMode 0 / 3)
# ----------------------------------------------------------------------------
def _fa_keep(q_len: int, kv_len: int, sparse_mode: int) -> np.ndarray:
    """Boolean [q_len, kv_len] mask of kept (query, key) pairs: sparseMode 0 keeps
    everything, sparseMode 3 keeps j <= i + kv_len - q_len (bottom-right causal)."""
    i = np.arange(q_len)[:, None]
    j = np.arange(kv_len)[None, :]
    if sparse_mode == 0:
        return np.ones((q_len, kv_len), bool)
    return j <= i + (kv_len - q_len)


def fa_forward(q, k, v, cu_seqlens_q, cu_seqlens_kv, scale: float, sparse_mode: int, dtype=np.float64):
    """Forward of aclnnFlashAttentionUnpaddingScoreGrad's attention (计算公式,
    keepProb = 1, no pse): q [T1, Nq, D], k/v [T2, Nkv, D] (TND), query head h
    reads kv head h // (Nq/Nkv).  Returns out [T1, Nq, D] and softmaxMax /
    softmaxSum in the page's [T1, Nq, 8] layout (8 equal copies)."""
    q, k, v = (_as(a, dtype) for a in (q, k, v))
    T1, Nq, _ = q.shape
    Nkv = k.shape[1]
    g = Nq // Nkv
    out = np.zeros((T1, Nq, v.shape[2]), dtype)
    smax = np.zeros((T1, Nq), dtype)
    ssum = np.zeros((T1, Nq), dtype)
    for sp in make_spans(LAYOUT_TND, len(cu_seqlens_q), 0, 0, cu_seqlens_q, cu_seqlens_kv):
        if sp.q_len == 0:
            continue
        keep = _fa_keep(sp.q_len, sp.kv_len, sparse_mode)
        qs = slice(sp.q_start, sp.q_start + sp.q_len)
        ks = slice(sp.kv_start, sp.kv_start + sp.kv_len)
        for h in range(Nq):
            s = scale * (q[qs, h] @ k[ks, h // g].T)
            s = np.where(keep, s, -np.inf)
            m = s.max(axis=1)
            has = np.isfinite(m)
            m = np.where(has, m, 0.0)
            e = np.where(keep, np.exp(s - m[:, None]), 0.0)
            l = e.sum(axis=1)
            w = e / np.where(l == 0, 1.0, l)[:, None]
            out[qs, h] = w @ v[ks, h // g]
            smax[qs, h] = m
            ssum[qs, h] = l
    rep = lambda a: np.repeat(a[:, :, None], 8, axis=2)
    return out, rep(smax), rep(ssum)


def fa_backward(q, k, v, dy, softmax_max, softmax_sum, attention_in, cu_seqlens_q, cu_seqlens_kv,
                scale: float, sparse_mode: int, dtype=np.float64):
    """dq, dk, dv of aclnnFlashAttentionUnpaddingScoreGrad (计算公式):
    P = exp(S - softmaxMax)/softmaxSum with S = scale*Q.K^T (kept pairs only),
    dV = P^T.dY, dS = P o (dY.V^T - rowsum(dY o attentionIn)),
    dQ = scale*dS.K, dK = scale*dS^T.Q; kv-head gradients sum over their query
    heads.  softmaxMax/softmaxSum are [T1, Nq, 8]; lane 0 is read."""
    q, k, v, dy, attention_in = (_as(a, dtype) for a in (q, k, v, dy, attention_in))
    m_all = _as(softmax_max, dtype)[:, :, 0]
    l_all = _as(softmax_sum, dtype)[:, :, 0]
    T1, Nq, _ = q.shape
    Nkv = k.shape[1]
    g = Nq // Nkv
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for sp in make_spans(LAYOUT_TND, len(cu_seqlens_q), 0, 0, cu_seqlens_q, cu_seqlens_kv):
        if sp.q_len == 0 or sp.kv_len == 0:
            continue
        keep = _fa_keep(sp.q_len, sp.kv_len, sparse_mode)
        qs = slice(sp.q_start, sp.q_start + sp.q_len)
        ks = slice(sp.kv_start, sp.kv_start + sp.kv_len)
        for h in range(Nq):
            hk = h // g
            s = scale * (q[qs, h] @ k[ks, hk].T)
            l = l_all[qs, h]
            inv_l = np.where(l == 0, 0.0, 1.0 / np.where(l == 0, 1.0, l))
            p = np.where(keep, np.exp(np.where(keep, s, 0.0) - m_all[qs, h][:, None]), 0.0) * inv_l[:, None]
            dv[ks, hk] += p.T @ dy[qs, h]
            dp = dy[qs, h] @ v[ks, hk].T
            dsum = (dy[qs, h] * attention_in[qs, h]).sum(axis=1)
            ds = p * (dp - dsum[:, None])
            dq[qs, h] = scale * (ds @ k[ks, hk])
            dk[ks, hk] += scale * (ds.T @ q[qs, h])
    return dq, dk, dv


def sfa_flops(indices, block_size: int, sparse_mode: int, layout: str, B: int, S1: int, S2: int, N1: int,
              D: int = 512, Dr: int = 64, seqlens_q=None, seqlens_kv=None) -> int:
    """Algorithmic backward FLOPs: 2*(S + dP + dV + dQ~ + dK~) contraction lengths
    per valid (token, head, key) triple, i.e. 2*(3*(D+Dr) + 2*D) = 5504 at D=512."""
    per = 2 * (3 * (D + Dr) + 2 * D)
    n = 0
    for sp in make_spans(layout, B, S1, S2, seqlens_q, seqlens_kv):
        for pos in range(sp.q_len):
            n += len(selected_rows(np.asarray(indices[sp.q_start + pos]), block_size, pos, sp.q_len,
                                   sp.kv_len, sparse_mode))
    return n * N1 * per
