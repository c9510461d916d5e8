"""Plain CPU oracle for the dense lightning-indexer gradient with its fused KL loss.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or run
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline``
/ ``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the
CUDA library; both sides only consume the same seeded inputs from ``workloads``.

Source: DenseLightningIndexerGradKLLoss (gitcode ops-transformer README,
"attention/dense_lightning_indexer_grad_kl_loss"), section 功能说明 (function
description), formulas 1-4, and 参数说明 (parameters).  Per query token t, over
the key rows j it may see (the page's K~_{:t,:}: sparseMode 3 keeps
j <= pos + S2_b - S1_b, sparseMode 0 keeps the whole sequence):

  S_tgj   = q~I[t,g] . K~I[j]                          indexer scores, G heads
  I_tj    = sum_g W[t,g] * ReLU(S_tgj)                 formula 1 (top-k value)
  P_thj   = exp(scale * Q~[t,h].K~[j] - softmaxMax[t,h]) / softmaxSum[t,h]
  p_tj    = sum_h P_thj / N1                           target distribution (formula 3 text)
  sI_tj   = exp(I_tj - softmaxMaxIndex[t]) / softmaxSumIndex[t]
  loss    = sum_t sum_j p_tj * (log p_tj - log sI_tj)  formula 3 (KL divergence)
  dI_tj   = sI_tj - p_tj                               formula 4
  dW[t,g] = sum_j dI_tj * ReLU(S_tgj)
  dS_tgj  = dI_tj * W[t,g] * [S_tgj > 0]
  dq~I[t,g] = sum_j dS_tgj * K~I[j]
  dK~I[j]  += sum_{t,g} dS_tgj * q~I[t,g]

with Q~ = [query || queryRope], K~ = [key || keyRope] (the main attention's MLA
shape, one key head) and q~I / K~I = queryIndex / keyIndex (one key head).

Readings taken where the page is silent (each is listed in the repository's
design notes):

* the target distribution sums the main attention's per-head softmax
  probabilities over the N1 heads and L1-normalises along the keys; with each
  head's probabilities summing to 1 that normalisation is a division by N1,
  which is what this oracle does (the statistics are used as given);
* the main attention's probabilities use softmaxMax / softmaxSum exactly as the
  sparse attention backward does (max of the scaled scores, sum of
  exp(scaled - max)); a softmaxSum of 0 gives P = 0;
* softmax(I) uses softmaxMaxIndex / softmaxSumIndex as given, one value per
  query token (the max of I_t and the sum of exp(I_t - max));
* the indexer scores carry no scale factor (formula 1 prints none);
* p log p is 0 where p = 0; the loss is the sum over tokens (one fp32 scalar);
* a token with no visible key contributes nothing (zero dq~I and dW rows);
* layouts, sequence lengths and sparseMode follow the sparse attention reading
  (BSND per-batch lengths, TND cumulative end offsets).

Parity status: pinned by ``tests/test_indexer_oracle_pins.py`` (finite
differences of the loss, a torch fp64 autograd special case built on
``torch.nn.functional.kl_div``, and the zero-divergence case).
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np

from .sfa_oracle import make_spans


def visible_keys(pos: int, q_len: int, kv_len: int, sparse_mode: int) -> int:
    """Number of leading key rows of the span that query position ``pos`` sees
    (the page's K~_{:t,:}; sparseMode 3 is the causal lower triangle aligned at
    the right vertex, as in the sparse attention backward)."""
    if sparse_mode == 3:
        return max(0, min(kv_len, pos + 1 + kv_len - q_len))
    return kv_len


def indexer_scores(q_index, k_index, weights, t: int, kv_start: int, n: int, dtype=np.float64):
    """S [G, n] and I [n] of query token t over key rows [kv_start, kv_start + n):
    formula 1, I = W_t . ReLU(q~I_t . K~I^T)."""
    qi = np.asarray(q_index[t], dtype)                 # [G, Di]
    ki = np.asarray(k_index[kv_start:kv_start + n], dtype)  # [n, Di]
    s = qi @ ki.T
    w = np.asarray(weights[t], dtype)                  # [G]
    return s, w @ np.maximum(s, 0.0)


def indexer_softmax_stats(q_index, k_index, weights, layout: str, B: int, S1: int, S2: int,
                          seqlens_q=None, seqlens_kv=None, sparse_mode: int = 3, dtype=np.float64):
    """softmaxMaxIndex / softmaxSumIndex [T1] that the indexer's forward would
    produce: the max over visible keys of I_t and the sum of exp(I_t - max)
    (0 and 0 for a token with no visible key)."""
    T1 = len(q_index)
    m = np.zeros(T1, dtype)
    l = np.zeros(T1, dtype)
    for sp in make_spans(layout, B, S1, S2, seqlens_q, seqlens_kv):
        for pos in range(sp.q_len):
            t = sp.q_start + pos
            n = visible_keys(pos, sp.q_len, sp.kv_len, sparse_mode)
            if n == 0:
                continue
            _, i = indexer_scores(q_index, k_index, weights, t, sp.kv_start, n, dtype)
            m[t] = i.max()
            l[t] = np.exp(i - m[t]).sum()
    return m, l


def indexer_kl_grad(q, k, q_index, k_index, weights, softmax_max, softmax_sum, softmax_max_index,
                    softmax_sum_index, q_rope, k_rope, scale: float, layout: str, B: int, S1: int, S2: int,
                    seqlens_q=None, seqlens_kv=None, sparse_mode: int = 3, dtype=np.float64, tokens=None):
    """dQueryIndex [T1, G, Di], dKeyIndex [T2, Di], dWeights [T1, G], loss (scalar)
    and the per-token losses [T1], following formulas 1-4 of the page written
    out per token (see the module docstring).

    q: [T1, N1, D], k: [T2, D], q_rope: [T1, N1, Dr], k_rope: [T2, Dr],
    q_index: [T1, G, Di], k_index: [T2, Di], weights: [T1, G],
    softmax_max / softmax_sum: [T1, N1], softmax_*_index: [T1].  ``tokens``
    restricts the sums to a subset of query rows (the dKeyIndex sum then only
    holds their contributions; the other query-side rows stay zero).
    """
    T1 = len(q)
    T2 = len(k)
    sel = None if tokens is None else set(int(t) for t in tokens)
    G, Di = np.asarray(q_index[0 if sel is None else min(sel)]).shape
    kt_all = np.concatenate([np.asarray(k, dtype), np.asarray(k_rope, dtype)], axis=1)  # [T2, D + Dr]
    ki_all = np.asarray(k_index, dtype)
    dq_index = np.zeros((T1, G, Di), dtype)
    dk_index = np.zeros((T2, Di), dtype)
    d_weights = np.zeros((T1, G), dtype)
    loss_t = np.zeros(T1, dtype)
    for sp in make_spans(layout, B, S1, S2, seqlens_q, seqlens_kv):
        for pos in range(sp.q_len):
            t = sp.q_start + pos
            if sel is not None and t not in sel:
                continue
            n = visible_keys(pos, sp.q_len, sp.kv_len, sparse_mode)
            if n == 0:
                continue
            rows = slice(sp.kv_start, sp.kv_start + n)
            # main attention probabilities with the given statistics, summed over heads
            qt = np.concatenate([np.asarray(q[t], dtype), np.asarray(q_rope[t], dtype)], axis=1)  # [N1, D + Dr]
            N1 = qt.shape[0]
            m = np.asarray(softmax_max[t], dtype)[:, None]
            l = np.asarray(softmax_sum[t], dtype)[:, None]
            prob = np.where(l > 0, np.exp(scale * (qt @ kt_all[rows].T) - m) / np.where(l > 0, l, 1.0), 0.0)
            p = prob.sum(axis=0) / N1                                             # [n]
            # indexer distribution with the given statistics
            s, i = indexer_scores(q_index, k_index, weights, t, sp.kv_start, n, dtype)
            mi = float(np.asarray(softmax_max_index[t]).reshape(-1)[0])
            li = float(np.asarray(softmax_sum_index[t]).reshape(-1)[0])
            log_si = (i - mi) - np.log(li) if li > 0 else np.full(n, -np.inf)
            si = np.exp(log_si)
            # KL(p || softmax(I)) with 0 log 0 = 0
            pos_p = p > 0
            loss_t[t] = np.sum(p[pos_p] * (np.log(p[pos_p]) - log_si[pos_p]))
            di = si - p                                                           # formula 4
            w = np.asarray(weights[t], dtype)
            d_weights[t] = np.maximum(s, 0.0) @ di                               # dW = dI . ReLU(S)^T
            ds = di[None, :] * w[:, None] * (s > 0)                              # [G, n]
            dq_index[t] = ds @ ki_all[rows]                                       # dq~I = dS . K~I
            dk_index[rows] += ds.T @ np.asarray(q_index[t], dtype)               # dK~I += dS^T . q~I
    return dq_index, dk_index, d_weights, float(loss_t.sum()), loss_t


def indexer_kl_grad_problem(p, softmax_max, softmax_sum, softmax_max_index, softmax_sum_index,
                            dtype=np.float64, tokens=None):
    """``indexer_kl_grad`` on a workloads.IndexerProblem."""
    return indexer_kl_grad(p.q, p.k, p.q_index, p.k_index, p.weights, softmax_max, softmax_sum,
                           softmax_max_index, softmax_sum_index, p.q_rope, p.k_rope, p.scale, p.layout, p.B,
                           p.S1, p.S2, p.seqlens_q, p.seqlens_kv, p.sparse_mode, dtype=dtype, tokens=tokens)
