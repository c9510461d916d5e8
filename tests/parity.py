"""Helpers shared by the GPU parity tests: move a workload to the device in the
library's layouts, run the library through its Python binding, run the oracle
on the same values, and compare with the stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

from oracle import sfa_oracle as O
from workloads import Problem, FAProblem

# bf16 outputs: max|err| <= 2e-2 * max|ref| and cosine >= 0.9999 per tensor
REL_TOL = 2e-2
COS_TOL = 0.9999


def assert_close(name: str, got, ref, rel: float = REL_TOL, cos: float = COS_TOL):
    got = np.asarray(got, np.float64).ravel()
    ref = np.asarray(ref, np.float64).ravel()
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{name}: non-finite values"
    mref = np.abs(ref).max() if ref.size else 0.0
    if mref == 0.0:
        assert np.abs(got).max() == 0.0, f"{name}: reference is zero, got max {np.abs(got).max()}"
        return
    err = np.abs(got - ref).max()
    c = float(got @ ref / (np.linalg.norm(got) * np.linalg.norm(ref) + 1e-300))
    assert err <= rel * mref, f"{name}: max|err| {err:.3e} > {rel} * max|ref| {mref:.3e} (cos {c:.6f})"
    assert c >= cos, f"{name}: cosine {c:.6f} < {cos}"


def _t(a, dtype, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device=dev, dtype=dtype)


class DevProblem:
    """Device tensors of a Problem in the library's layouts."""

    def __init__(self, p: Problem, dtype=torch.bfloat16, dev="cuda"):
        self.p = p
        self.dtype = dtype
        if p.layout == "BSND":
            qs = (p.B, p.S1, p.N1)
            ks = (p.B, p.S2, 1)
            ishape = (p.B, p.S1, 1, p.topk)
        else:
            qs = (p.T1, p.N1)
            ks = (p.T2, 1)
            ishape = (p.T1, 1, p.topk)
        self.qs, self.ks = qs, ks
        self.q = _t(p.q, dtype, dev).reshape(*qs, p.D)
        self.qr = _t(p.q_rope, dtype, dev).reshape(*qs, p.Dr)
        self.k = _t(p.k, dtype, dev).reshape(*ks, p.D)
        self.kr = _t(p.k_rope, dtype, dev).reshape(*ks, p.Dr)
        self.v = self.k if p.value_is_key else _t(p.v, dtype, dev).reshape(*ks, p.D)
        self.do = _t(p.dout, dtype, dev).reshape(*qs, p.D)
        self.idx = _t(p.indices, torch.int32, dev).reshape(ishape)
        self.sq = None if p.seqlens_q is None else _t(p.seqlens_q, torch.int32, dev)
        self.skv = None if p.seqlens_kv is None else _t(p.seqlens_kv, torch.int32, dev)
        self.out = self.smax = self.ssum = None

    def kw(self):
        p = self.p
        return dict(scale=p.scale, sparse_block_size=p.block_size, layout=p.layout, sparse_mode=p.sparse_mode,
                    actual_seq_lengths_q=self.sq, actual_seq_lengths_kv=self.skv)

    def set_forward(self, out, smax, ssum):
        """Use given O / stats (numpy, flattened [T1, N1, ...]) as the backward's inputs."""
        p = self.p
        self.out = _t(out, self.dtype, self.q.device).reshape(*self.qs, p.D)
        self.smax = _t(smax, torch.float32, self.q.device).reshape(*self.qs)
        self.ssum = _t(ssum, torch.float32, self.q.device).reshape(*self.qs)

    def forward_gpu(self):
        import sparse_attention_backward_sfa_b200 as S
        self.out, self.smax, self.ssum = S.sfa_fwd(self.q, self.k, self.v, self.idx, self.qr, self.kr, **self.kw())
        return self.out, self.smax, self.ssum

    def grad_gpu(self, deterministic=None, **extra):
        import sparse_attention_backward_sfa_b200 as S
        det = self.p.deterministic if deterministic is None else deterministic
        return S.sfa_grad(self.q, self.k, self.v, self.idx, self.do, self.out, self.smax, self.ssum, self.qr,
                          self.kr, deterministic=det, **self.kw(), **extra)

    def host_fwd_inputs(self):
        """O / stats as numpy (flattened) exactly as the device holds them."""
        p = self.p
        return (self.out.float().cpu().numpy().reshape(p.T1, p.N1, p.D),
                self.smax.cpu().numpy().reshape(p.T1, p.N1).astype(np.float64),
                self.ssum.cpu().numpy().reshape(p.T1, p.N1).astype(np.float64))


def oracle_forward(p: Problem, tokens=None):
    return O.sfa_forward(p.q, p.k, p.value, p.indices, p.q_rope, p.k_rope, p.scale, p.block_size, p.sparse_mode,
                         p.layout, p.B, p.S1, p.S2, p.seqlens_q, p.seqlens_kv, tokens=tokens)


def oracle_backward(p: Problem, out, smax, ssum, tokens=None, dtype=np.float64):
    return O.sfa_backward(p.q, p.k, p.value, p.indices, p.dout, out, smax, ssum, p.q_rope, p.k_rope, p.scale,
                          p.block_size, p.sparse_mode, p.layout, p.B, p.S1, p.S2, p.seqlens_q, p.seqlens_kv,
                          tokens=tokens, dtype=dtype)


def round_bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def prepare_oracle_forward(p: Problem, dp: DevProblem):
    """Workload-1 recipe: O and stats from the oracle forward; O rounded to the
    16-bit input type, stats to fp32, then handed to both sides."""
    out, m, l = oracle_forward(p)
    out_q = round_bf16(out) if dp.dtype == torch.bfloat16 else np.asarray(out, np.float16).astype(np.float32)
    m32 = np.asarray(m, np.float32)
    l32 = np.asarray(l, np.float32)
    dp.set_forward(out_q, m32, l32)
    return out_q.astype(np.float64), m32.astype(np.float64), l32.astype(np.float64)


def grads_np(res, p: Problem):
    dq, dk, dv, dqr, dkr = (r.float().cpu().numpy() for r in res)
    return (dq.reshape(p.T1, p.N1, p.D), dk.reshape(p.T2, p.D), dv.reshape(p.T2, p.D),
            dqr.reshape(p.T1, p.N1, p.Dr), dkr.reshape(p.T2, p.Dr))


NAMES = ("dQuery", "dKey", "dValue", "dQueryRope", "dKeyRope")


def compare_grads(got, ref, tokens=None, what=""):
    """Compare the five gradients; with `tokens`, the oracle's dQuery rows are
    the sampled rows only (ascending) and the GPU rows are selected to match."""
    for i, (n, g, r) in enumerate(zip(NAMES, got, ref)):
        if tokens is not None and i in (0, 3):
            g = g[np.sort(np.asarray(tokens))]
        assert_close(f"{what}{n}", g, r)


class DevFA:
    def __init__(self, fp: FAProblem, dtype=torch.bfloat16, dev="cuda"):
        self.fp = fp
        self.q = _t(fp.q, dtype, dev)
        self.k = _t(fp.k, dtype, dev)
        self.v = _t(fp.v, dtype, dev)
        self.dy = _t(fp.dy, dtype, dev)
        self.dtype = dtype
        self.out = self.smax = self.ssum = None

    def forward_gpu(self):
        import sparse_attention_backward_sfa_b200 as S
        fp = self.fp
        self.out, self.smax, self.ssum = S.fa_fwd(self.q, self.k, self.v, fp.cu_seqlens_q, fp.cu_seqlens_kv,
                                                  scale=fp.scale, sparse_mode=fp.sparse_mode)
        return self.out, self.smax, self.ssum

    def grad_gpu(self, deterministic=False, **extra):
        import sparse_attention_backward_sfa_b200 as S
        fp = self.fp
        return S.fa_grad(self.q, self.k, self.v, self.dy, self.smax, self.ssum, self.out, fp.cu_seqlens_q,
                         fp.cu_seqlens_kv, scale=fp.scale, sparse_mode=fp.sparse_mode, deterministic=deterministic,
                         **extra)
