"""Seeded generators for the sparse-attention backward workloads.

The five workloads (sizes, distributions and index structure):

1. SFA, BSND, B=1, S1=128, S2=2048, N1=1, D=512, Dr=64, sparseMode 0, topk=1024,
   block 1: per token 1024 distinct rows uniform in [0, 2048), sorted.
2. Dense varlen FA, TND, sequences {512, 1024, 1536, 2048} (T=5120), N=16 heads,
   D=128, causal, scale 1/sqrt(128).
3. SFA, BSND, B=1, S1=S2=8192, N1=64, sparseMode 3, topk=2048, block 1: token t
   takes distinct rows uniform in [0, t] (all of them when t+1 <= 2048), random
   order, -1 padding at the tail; atomic.
4. SFA, TND, sequences {2048, 4096, 4096, 6144} (T=16384), N1=128, sparseMode 3,
   topk=1024 blocks of 16: distinct causal-valid block indices in random order,
   -1 padding; deterministic.
5. SFA, BSND, B=1, S1=S2=32768, N1=128, sparseMode 3, topk=8192, block 1:
   distinct causal-valid rows in random order, -1 padding; atomic.

q / k / q_rope / k_rope / dO (and FA's q/k/v/dY) are N(0, 1) rounded to bf16;
value is the same tensor as key.  O and the softmax statistics are not made
here: the caller runs a forward (oracle or GPU) on these inputs.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Dict, List, Optional

import numpy as np
import torch


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float data to bf16 (round-to-nearest-even) and return it as float32."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) of float data, rounding to nearest even."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


@dataclass
class Problem:
    """One sparse-attention backward problem in flattened form.

    BSND tensors are stored flattened: q [B*S1, N1, D], k [B*S2, D] (N2 = 1),
    indices [B*S1, topk].  TND tensors are [T1, ...] / [T2, ...] directly.
    """

    name: str
    layout: str  # "BSND" | "TND"
    B: int
    S1: int
    S2: int
    T1: int
    T2: int
    N1: int
    D: int
    Dr: int
    topk: int
    block_size: int
    sparse_mode: int
    deterministic: bool
    scale: float
    seqlens_q: Optional[np.ndarray]  # BSND: per-batch lengths or None; TND: cumulative ends
    seqlens_kv: Optional[np.ndarray]
    q: np.ndarray
    q_rope: np.ndarray
    k: np.ndarray
    k_rope: np.ndarray
    dout: np.ndarray
    indices: np.ndarray
    value_is_key: bool = True
    v: Optional[np.ndarray] = None
    out: Optional[np.ndarray] = None
    softmax_max: Optional[np.ndarray] = None
    softmax_sum: Optional[np.ndarray] = None
    meta: Dict = field(default_factory=dict)

    @property
    def value(self) -> np.ndarray:
        return self.k if self.value_is_key else self.v


@dataclass
class FAProblem:
    name: str
    cu_seqlens_q: np.ndarray  # cumulative end offsets, length B
    cu_seqlens_kv: np.ndarray
    Nq: int
    Nkv: int
    D: int
    scale: float
    sparse_mode: int
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    dy: np.ndarray
    out: Optional[np.ndarray] = None
    softmax_max: Optional[np.ndarray] = None
    softmax_sum: Optional[np.ndarray] = None


def _normal(rng, shape):
    return bf16_round(rng.standard_normal(shape, dtype=np.float32))


def _causal_distinct(rng: np.random.Generator, n_valid: np.ndarray, topk: int, chunk: int = 512) -> np.ndarray:
    """Row t: min(n_valid[t], topk) distinct values uniform in [0, n_valid[t]) in
    random order, then -1 padding."""
    T = len(n_valid)
    out = np.full((T, topk), -1, np.int32)
    hi = int(n_valid.max()) if T else 0
    for s in range(0, T, chunk):
        nv = n_valid[s:s + chunk]
        keys = rng.random((len(nv), hi), dtype=np.float32)
        keys[np.arange(hi)[None, :] >= nv[:, None]] = 2.0
        kk = min(topk, hi)
        part = np.argpartition(keys, kk - 1, axis=1)[:, :kk] if kk < hi else np.argsort(keys, axis=1)[:, :kk]
        part = rng.permuted(part, axis=1)
        take = np.minimum(nv, topk)
        # valid entries first (in random order), then -1
        vals = np.take_along_axis(keys, part, axis=1) < 1.5
        order = np.argsort(~vals, axis=1, kind="stable")
        part = np.take_along_axis(part, order, axis=1)
        part = np.where(np.arange(kk)[None, :] < take[:, None], part, -1)
        out[s:s + chunk, :kk] = part
    return out


def _scale(D, Dr):
    return 1.0 / math.sqrt(D + Dr)


def make_problem(cfg: int, seed: Optional[int] = None) -> Problem:
    """Workloads 1, 3, 4, 5 (see module docstring).  Seed defaults to 1000 + cfg."""
    rng = np.random.default_rng(1000 + cfg if seed is None else seed)
    D, Dr = 512, 64
    if cfg == 1:
        B, S1, S2, N1, topk, bs, mode, det = 1, 128, 2048, 1, 1024, 1, 0, False
        layout, sq, skv = "BSND", None, None
        T1, T2 = B * S1, B * S2
        idx = np.sort(np.stack([rng.choice(S2, topk, replace=False) for _ in range(T1)]), axis=1).astype(np.int32)
    elif cfg == 3:
        B, S1, S2, N1, topk, bs, mode, det = 1, 8192, 8192, 64, 2048, 1, 3, False
        layout, sq, skv = "BSND", None, None
        T1, T2 = B * S1, B * S2
        idx = _causal_distinct(rng, np.arange(1, S1 + 1), topk)
    elif cfg == 4:
        lens = [2048, 4096, 4096, 6144]
        B, N1, topk, bs, mode, det = 4, 128, 1024, 16, 3, True
        layout = "TND"
        cu = np.cumsum(lens).astype(np.int32)
        sq, skv = cu.copy(), cu.copy()
        T1 = T2 = int(cu[-1])
        S1 = S2 = 0
        nvalid = np.concatenate([np.arange(L) // bs + 1 for L in lens])
        idx = _causal_distinct(rng, nvalid, topk)
    elif cfg == 5:
        B, S1, S2, N1, topk, bs, mode, det = 1, 32768, 32768, 128, 8192, 1, 3, False
        layout, sq, skv = "BSND", None, None
        T1, T2 = B * S1, B * S2
        idx = _causal_distinct(rng, np.arange(1, S1 + 1), topk, chunk=256)
    else:
        raise ValueError(cfg)
    q = _normal(rng, (T1, N1, D))
    qr = _normal(rng, (T1, N1, Dr))
    k = _normal(rng, (T2, D))
    kr = _normal(rng, (T2, Dr))
    do = _normal(rng, (T1, N1, D))
    return Problem(f"cfg{cfg}", layout, B, S1, S2, T1, T2, N1, D, Dr, topk, bs, mode, det, _scale(D, Dr),
                   sq, skv, q, qr, k, kr, do, idx)


def make_fa_problem(seed: int = 1002, lens=(512, 1024, 1536, 2048), N: int = 16, Nkv: Optional[int] = None,
                    D: int = 128, sparse_mode: int = 3, kv_lens=None) -> FAProblem:
    """Workload 2 (dense varlen FA backward) or a smaller variant of it."""
    rng = np.random.default_rng(seed)
    Nkv = N if Nkv is None else Nkv
    cq = np.cumsum(lens).astype(np.int64)
    ck = np.cumsum(lens if kv_lens is None else kv_lens).astype(np.int64)
    T1, T2 = int(cq[-1]), int(ck[-1])
    q = _normal(rng, (T1, N, D))
    k = _normal(rng, (T2, Nkv, D))
    v = _normal(rng, (T2, Nkv, D))
    dy = _normal(rng, (T1, N, D))
    return FAProblem(f"fa{len(lens)}x{N}x{D}", cq, ck, N, Nkv, D, 1.0 / math.sqrt(D), sparse_mode, q, k, v, dy)


def tiny_problem(seed: int, layout: str = "BSND", B: int = 1, S1: int = 6, S2: int = 16, N1: int = 2,
                 D: int = 8, Dr: int = 4, topk: int = 4, block_size: int = 1, sparse_mode: int = 0,
                 seqlens_q=None, seqlens_kv=None, index_mode: str = "distinct", deterministic: bool = False,
                 value_is_key: bool = True, scale: Optional[float] = None, round_bf16: bool = True) -> Problem:
    """Small problem with general D / Dr for oracle pins and parity edge cases.

    index_mode:
      "distinct" - distinct blocks uniform over [0, ceil(S2_b/bs)), random order, -1 pad
      "causal"   - distinct causal-valid blocks (as in workloads 3-5), -1 pad
      "messy"    - anything: -1 anywhere, duplicates, blocks past S2_b, negative values
      "all"      - every block, in random order (dense special case)
    For TND, seqlens_q/kv are per-sequence lengths here and are returned cumulative.
    """
    rng = np.random.default_rng(seed)
    if layout == "TND":
        lq = np.asarray(seqlens_q, np.int64)
        lk = np.asarray(seqlens_kv if seqlens_kv is not None else seqlens_q, np.int64)
        B = len(lq)
        T1, T2 = int(lq.sum()), int(lk.sum())
        sq, skv = np.cumsum(lq).astype(np.int32), np.cumsum(lk).astype(np.int32)
        q_len_of = np.repeat(lq, lq)
        pos_of = np.concatenate([np.arange(n) for n in lq]) if T1 else np.zeros(0, np.int64)
        kv_len_of = np.repeat(lk, lq)
        S1 = S2 = 0
    else:
        T1, T2 = B * S1, B * S2
        lq = np.full(B, S1) if seqlens_q is None else np.asarray(seqlens_q)
        lk = np.full(B, S2) if seqlens_kv is None else np.asarray(seqlens_kv)
        sq = None if seqlens_q is None else np.asarray(seqlens_q, np.int32)
        skv = None if seqlens_kv is None else np.asarray(seqlens_kv, np.int32)
        q_len_of = np.repeat(lq, S1)
        kv_len_of = np.repeat(lk, S1)
        pos_of = np.tile(np.arange(S1), B)
    idx = np.full((T1, topk), -1, np.int32)
    for t in range(T1):
        nblk = -(-int(kv_len_of[t]) // block_size)
        if index_mode == "distinct":
            c = rng.permutation(max(nblk, 0))[:topk]
        elif index_mode == "causal":
            lim = int(pos_of[t]) + int(kv_len_of[t]) - int(q_len_of[t])
            nvb = 0 if lim < 0 else min(nblk, lim // block_size + 1)
            c = rng.permutation(nvb)[:topk]
        elif index_mode == "all":
            c = rng.permutation(nblk)[:topk]
        elif index_mode == "messy":
            c = rng.integers(-2, nblk + 2, size=topk)
        else:
            raise ValueError(index_mode)
        idx[t, :len(c)] = c
    rnd = bf16_round if round_bf16 else (lambda a: a.astype(np.float64))
    q = rnd(rng.standard_normal((T1, N1, D)))
    qr = rnd(rng.standard_normal((T1, N1, Dr)))
    k = rnd(rng.standard_normal((T2, D)))
    kr = rnd(rng.standard_normal((T2, Dr)))
    do = rnd(rng.standard_normal((T1, N1, D)))
    v = None if value_is_key else rnd(rng.standard_normal((T2, D)))
    sc = 1.0 / math.sqrt(D + Dr) if scale is None else scale
    return Problem(f"tiny{seed}", layout, B, S1, S2, T1, T2, N1, D, Dr, topk, block_size, sparse_mode,
                   deterministic, sc, sq, skv, q, qr, k, kr, do, idx, value_is_key, v)


def subproblem(p: Problem, n_tokens: int = 256, seed: Optional[int] = None):
    """Seeded sample of query rows (among rows that are inside their batch's
    valid length) and a copy of the problem whose dO is zero on every other row.
    A zero dO row contributes exactly nothing to any gradient, so the full-size
    run of the copy equals the sub-problem made of the sampled rows."""
    rng = np.random.default_rng((p.meta.get("seed", 0) + 1) if seed is None else seed)
    if p.layout == "TND":
        valid = np.arange(p.T1)
    else:
        lq = np.full(p.B, p.S1) if p.seqlens_q is None else np.asarray(p.seqlens_q)
        valid = np.concatenate([b * p.S1 + np.arange(lq[b]) for b in range(p.B)])
    toks = np.sort(rng.choice(valid, size=min(n_tokens, len(valid)), replace=False))
    d2 = np.zeros_like(p.dout)
    d2[toks] = p.dout[toks]
    return toks, replace(p, dout=d2)


WORKLOADS = {
    1: "sfa_bsnd_s128x2048_n1_topk1024_bs1_mode0",
    2: "fa_tnd_512-1024-1536-2048_n16_d128_causal",
    3: "sfa_bsnd_s8192_n64_topk2048_bs1_causal_atomic",
    4: "sfa_tnd_2048-4096-4096-6144_n128_topk1024x16_causal_deterministic",
    5: "sfa_bsnd_s32768_n128_topk8192_bs1_causal_atomic",
}


# ---------------------------------------------------------------------------
# Device-side generation of the large workloads (3, 4, 5)
# ---------------------------------------------------------------------------
def _dev_causal_distinct(gen: torch.Generator, n_valid: torch.Tensor, topk: int, chunk: int) -> torch.Tensor:
    """Row t: min(n_valid[t], topk) distinct values uniform in [0, n_valid[t]),
    random order, then -1 padding (same distribution as the host generator)."""
    T = n_valid.numel()
    dev = n_valid.device
    hi = int(n_valid.max().item())
    kk = min(topk, hi)
    out = torch.full((T, topk), -1, dtype=torch.int32, device=dev)
    ar = torch.arange(hi, device=dev)[None, :]
    for s in range(0, T, chunk):
        nv = n_valid[s:s + chunk]
        keys = torch.rand((nv.numel(), hi), generator=gen, device=dev)
        keys.masked_fill_(ar >= nv[:, None], 2.0)
        val, pos = torch.topk(keys, kk, dim=1, largest=False, sorted=True)
        pos = torch.where(val < 1.5, pos, torch.full_like(pos, -1))
        out[s:s + chunk, :kk] = pos.to(torch.int32)
    return out


def make_device_problem(cfg: int, device="cuda", seed: Optional[int] = None, seqs=None) -> Problem:
    """Workloads 3, 4, 5 generated directly on the device as torch tensors in the
    library's layouts (q [B,S1,N1,D] or [T1,N1,D], key [..,1,D], indices
    [..,1,topk]); value is key.  Seed defaults to 2000 + cfg.  `seqs` replaces
    workload 4's sequence lengths, or workload 5's sequence length S (topk scaled
    with it, 8192 * S / 32768, so every row keeps its share of selected keys): a
    smaller case of the same shape, used for profiling captures."""
    gen = torch.Generator(device=device)
    gen.manual_seed(2000 + cfg if seed is None else seed)
    D, Dr = 512, 64
    if cfg == 3:
        B, S, N1, topk, bs = 1, 8192, 64, 2048, 1
        layout, lens = "BSND", None
    elif cfg == 4:
        lens = [2048, 4096, 4096, 6144] if seqs is None else [int(x) for x in seqs]
        B, N1, topk, bs = len(lens), 128, 1024, 16
        layout = "TND"
    elif cfg == 5:
        B, S, N1, topk, bs = 1, 32768, 128, 8192, 1
        if seqs is not None:
            S = int(seqs[0])
            topk = max(1, 8192 * S // 32768)
        layout, lens = "BSND", None
    else:
        raise ValueError(cfg)
    if layout == "BSND":
        T1 = T2 = B * S
        S1 = S2 = S
        nvalid = torch.arange(1, S + 1, device=device).repeat(B)
        sq = skv = None
        qs, ks, ish = (B, S, N1), (B, S, 1), (B, S, 1, topk)
    else:
        T1 = T2 = int(sum(lens))
        S1 = S2 = 0
        nvalid = torch.cat([torch.arange(L, device=device) // bs + 1 for L in lens])
        cu = torch.tensor(np.cumsum(lens), dtype=torch.int32, device=device)
        sq = skv = cu
        qs, ks, ish = (T1, N1), (T2, 1), (T1, 1, topk)
    idx = _dev_causal_distinct(gen, nvalid, topk, chunk=max(1, (1 << 25) // int(nvalid.max().item()))).reshape(ish)

    def rnd(*shape):
        return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)

    q = rnd(*qs, D)
    qr = rnd(*qs, Dr)
    k = rnd(*ks, D)
    kr = rnd(*ks, Dr)
    do = rnd(*qs, D)
    det = cfg == 4
    return Problem(f"cfg{cfg}", layout, B, S1, S2, T1, T2, N1, D, Dr, topk, bs, 3, det, _scale(D, Dr), sq, skv,
                   q, qr, k, kr, do, idx, meta={"seed": 2000 + cfg if seed is None else seed, "device": True})


class RowView:
    """Row access t -> numpy row for a subset of rows of a large device tensor,
    so the oracle can run on sampled query rows without a full host copy."""

    def __init__(self, tensor: torch.Tensor, rows, flat_rows: int):
        flat = tensor.reshape(flat_rows, -1)
        self._shape = tensor.shape[tensor.dim() - _row_rank(tensor, flat_rows):]
        rows = sorted(int(r) for r in rows)
        sel = flat[torch.tensor(rows, device=tensor.device, dtype=torch.long)]
        sel = (sel.float() if sel.is_floating_point() else sel).cpu().numpy()
        self._rows = {r: sel[i].reshape(self._shape) for i, r in enumerate(rows)}
        self._n = flat_rows

    def __len__(self):
        return self._n

    def __getitem__(self, t):
        return self._rows[int(t)]


def _row_rank(tensor: torch.Tensor, flat_rows: int) -> int:
    """Number of trailing dims that make up one flattened row."""
    n = 1
    for r in range(tensor.dim() - 1, -1, -1):
        lead = int(np.prod(tensor.shape[:r])) if r else 1
        if lead == flat_rows:
            return tensor.dim() - r
    raise ValueError("row count does not match a leading product of the shape")


# ---------------------------------------------------------------------------
# Dense lightning-indexer gradient with KL loss: inputs
# ---------------------------------------------------------------------------
INDEXER_WORKLOAD = "indexer_kl_tnd_2048-4096-4096-6144_n128_g64_d128_causal"


@dataclass
class IndexerProblem:
    """Inputs of the dense lightning-indexer gradient (flattened like Problem):
    q [T1, N1, D], q_rope [T1, N1, Dr], k [T2, D], k_rope [T2, Dr] (the main
    attention, one key head), q_index [T1, G, Di], k_index [T2, Di] (one indexer
    key head), weights [T1, G].  The softmax statistics of both distributions are
    not made here: the caller derives them (oracle or GPU forward)."""

    name: str
    layout: str
    B: int
    S1: int
    S2: int
    T1: int
    T2: int
    N1: int
    G: int
    Di: int
    D: int
    Dr: int
    sparse_mode: int
    scale: float
    seqlens_q: Optional[np.ndarray]  # BSND: per-batch lengths or None; TND: cumulative ends
    seqlens_kv: Optional[np.ndarray]
    q: np.ndarray
    q_rope: np.ndarray
    k: np.ndarray
    k_rope: np.ndarray
    q_index: np.ndarray
    k_index: np.ndarray
    weights: np.ndarray
    meta: Dict = field(default_factory=dict)


def indexer_problem(seed: int, layout: str = "TND", B: int = 1, S1: int = 0, S2: int = 0, seqlens_q=None,
                    seqlens_kv=None, N1: int = 4, G: int = 4, Di: int = 8, D: int = 8, Dr: int = 4,
                    sparse_mode: int = 3, scale: Optional[float] = None, round_bf16: bool = True) -> IndexerProblem:
    """Small or medium indexer-gradient problem.  q / k / q_rope / k_rope /
    q_index / k_index are N(0, 1); weights are N(0, 1) / sqrt(G); all rounded to
    bf16 unless round_bf16 is False.  For TND, seqlens_q/kv are per-sequence
    lengths here and are returned cumulative (int64)."""
    rng = np.random.default_rng(seed)
    if layout == "TND":
        lq = np.asarray(seqlens_q, np.int64)
        lk = np.asarray(seqlens_kv if seqlens_kv is not None else seqlens_q, np.int64)
        B = len(lq)
        T1, T2 = int(lq.sum()), int(lk.sum())
        sq, skv = np.cumsum(lq).astype(np.int64), np.cumsum(lk).astype(np.int64)
        S1 = S2 = 0
    else:
        T1, T2 = B * S1, B * S2
        sq = None if seqlens_q is None else np.asarray(seqlens_q, np.int64)
        skv = None if seqlens_kv is None else np.asarray(seqlens_kv, np.int64)
    rnd = bf16_round if round_bf16 else (lambda a: a.astype(np.float64))
    q = rnd(rng.standard_normal((T1, N1, D)))
    qr = rnd(rng.standard_normal((T1, N1, Dr)))
    k = rnd(rng.standard_normal((T2, D)))
    kr = rnd(rng.standard_normal((T2, Dr)))
    qi = rnd(rng.standard_normal((T1, G, Di)))
    ki = rnd(rng.standard_normal((T2, Di)))
    w = rnd(rng.standard_normal((T1, G)) / math.sqrt(G))
    sc = 1.0 / math.sqrt(D + Dr) if scale is None else scale
    return IndexerProblem(f"indexer{seed}", layout, B, S1, S2, T1, T2, N1, G, Di, D, Dr, sparse_mode, sc, sq, skv,
                          q, qr, k, kr, qi, ki, w, meta={"seed": seed})


def make_device_indexer_problem(device="cuda", seed: int = 3000, seqs=(2048, 4096, 4096, 6144), N1: int = 128,
                                G: int = 64, Di: int = 128) -> IndexerProblem:
    """The indexer-gradient benchmark workload generated on the device (torch
    bf16 tensors in the library's TND layouts: q [T1,N1,512], key [T2,1,512],
    q_index [T1,G,Di], k_index [T2,1,Di], weights [T1,G]); causal (mode 3)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    D, Dr = 512, 64
    lens = [int(x) for x in seqs]
    T = int(sum(lens))
    cu = torch.tensor(np.cumsum(lens), dtype=torch.int64, device=device)

    def rnd(*shape, s=1.0):
        return (torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * s).to(torch.bfloat16)

    return IndexerProblem(INDEXER_WORKLOAD, "TND", len(lens), 0, 0, T, T, N1, G, Di, D, Dr, 3, _scale(D, Dr), cu, cu,
                          rnd(T, N1, D), rnd(T, N1, Dr), rnd(T, 1, D), rnd(T, 1, Dr), rnd(T, G, Di), rnd(T, 1, Di),
                          rnd(T, G, s=1.0 / math.sqrt(G)), meta={"seed": seed, "device": True})
