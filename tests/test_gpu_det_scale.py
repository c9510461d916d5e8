"""Deterministic mode at small gradient scales (GPU).

The deterministic key-side sums are 64-bit fixed point on a per-call power-of-two
grid that follows max|dOut| (SparseFlashAttentionGrad README, 确定性计算, asks for
run-to-run identical results; the tolerance of every output still has to hold).
These cases scale dOut by 1e-4 and 1e-8, where a fixed absolute grid would round
most contributions away, and compare every deterministic path with the oracle:
the fused tensor-core backward (N1 = 128 and 64), the CUDA-core backward, the
dense FA backward, the row-range (sharded) path and the pipelined host path.
A power-of-two scale of dOut must scale the deterministic results exactly.
"""
import numpy as np
import pytest
import torch

from oracle import sfa_oracle as O
from workloads import make_fa_problem, tiny_problem
from parity import (DevFA, DevProblem, assert_close, compare_grads, grads_np, oracle_backward,
                    prepare_oracle_forward, round_bf16)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_backward_sfa_b200 import build
    build.build()


PATHS = {
    # fused tcgen05 backward, N1 = 128, block-sparse causal rows (several tiles, ragged tail)
    "fused_n128": dict(layout="TND", seqlens_q=[150, 40], seqlens_kv=[300, 40], N1=128, topk=24, block_size=16,
                       sparse_mode=3, index_mode="causal"),
    # fused tcgen05 backward, N1 = 64, row gathers
    "fused_n64": dict(layout="BSND", B=1, S1=9, S2=400, N1=64, topk=300, block_size=1, sparse_mode=0),
    # CUDA-core backward (N1 below the fused sizes)
    "generic_n8": dict(layout="BSND", B=2, S1=7, S2=90, N1=8, topk=40, block_size=2, sparse_mode=3,
                       index_mode="causal"),
}


def scaled_problem(case, s, seed=907):
    """The case's problem with dOut multiplied by s (then rounded to bf16, the value both sides use)."""
    p = tiny_problem(seed, D=512, Dr=64, **PATHS[case])
    p.dout = round_bf16(np.asarray(p.dout, np.float64) * s).astype(np.float64)
    return p


@pytest.mark.parametrize("case", sorted(PATHS))
@pytest.mark.parametrize("s", [1e-4, 1e-8])
def test_deterministic_small_gradient_matches_oracle(case, s):
    p = scaled_problem(case, s)
    dp = DevProblem(p)
    out, m, l = prepare_oracle_forward(p, dp)
    got = grads_np(dp.grad_gpu(deterministic=True), p)
    compare_grads(got, oracle_backward(p, out, m, l), what=f"{case}/dO x {s}/")


@pytest.mark.parametrize("case", sorted(PATHS))
def test_deterministic_power_of_two_scale_is_exact(case):
    """dOut * 2^-27 gives exactly 2^-27 times the unscaled deterministic results (bit for bit)."""
    p = tiny_problem(911, D=512, Dr=64, **PATHS[case])
    dp = DevProblem(p)
    prepare_oracle_forward(p, dp)
    base = [x.float() for x in dp.grad_gpu(deterministic=True)]
    dp.do = (dp.do.float() * 2.0 ** -27).to(dp.do.dtype)
    small = [x.float() for x in dp.grad_gpu(deterministic=True)]
    for name, a, b in zip(("dQuery", "dKey", "dValue", "dQueryRope", "dKeyRope"), base, small):
        assert torch.equal(a * 2.0 ** -27, b), f"{case}: {name} is not exactly scaled"


@pytest.mark.parametrize("s", [1e-4, 1e-8])
def test_fa_deterministic_small_gradient(s):
    fp = make_fa_problem(seed=913, lens=(37, 1, 64), N=8, Nkv=2, D=128, sparse_mode=3, kv_lens=(50, 9, 64))
    fp.dy = round_bf16(np.asarray(fp.dy, np.float64) * s).astype(np.float64)
    d = DevFA(fp)
    d.forward_gpu()
    out = d.out.float().cpu().numpy()
    sm = d.smax.cpu().numpy().astype(np.float64)
    ss = d.ssum.cpu().numpy().astype(np.float64)
    dq, dk, dv = (x.float().cpu().numpy() for x in d.grad_gpu(deterministic=True))
    rq, rk, rv = O.fa_backward(fp.q, fp.k, fp.v, fp.dy, sm, ss, out, fp.cu_seqlens_q, fp.cu_seqlens_kv, fp.scale,
                               fp.sparse_mode)
    assert_close(f"fa dq (dY x {s})", dq, rq)
    assert_close(f"fa dk (dY x {s})", dk, rk)
    assert_close(f"fa dv (dY x {s})", dv, rv)


@pytest.mark.parametrize("case", ["fused_n128", "generic_n8"])
def test_rows_path_small_gradient(case):
    """Three row ranges (boundaries on even rows), each into its own accumulator, summed (what the
    ranks' all-reduce does), with the grid from the max of the ranges' max|dOut|: bit-identical
    to sfa_grad and within the tolerance of the oracle at dOut x 1e-8."""
    import sparse_attention_backward_sfa_b200 as S
    p = scaled_problem(case, 1e-8, seed=919)
    dp = DevProblem(p)
    out, m, l = prepare_oracle_forward(p, dp)
    full = dp.grad_gpu(deterministic=True)
    kw = dp.kw()
    T1 = p.T1
    a, b = 2 * (T1 // 6), 2 * (T1 // 3) + 2  # even boundaries: the pairs of rows of the whole call
    ranges = [(0, a), (a, b), (b, T1)]
    dmax = torch.zeros(1, dtype=torch.float32, device="cuda")
    for rb, re_ in ranges:
        S.dout_absmax(dp.do, dp.q, dp.k, dp.qr, dp.idx, layout=p.layout, row_begin=rb, row_end=re_,
                      actual_seq_lengths_q=dp.sq, into=dmax)
    dq = torch.zeros_like(dp.q)
    dqr = torch.zeros_like(dp.qr)
    accs = []
    for rb, re_ in ranges:
        acc = S.sfa_dkv_accumulator(dp.q, dp.k, dp.qr, dp.idx, layout=p.layout, deterministic=True,
                                    actual_seq_lengths_q=dp.sq)
        S.sfa_grad_rows(dp.q, dp.k, dp.v, dp.idx, dp.do, dp.out, dp.smax, dp.ssum, dp.qr, dp.kr, row_begin=rb,
                        row_end=re_, dkv_accum=acc, deterministic=True, dout_absmax=dmax, d_query=dq,
                        d_query_rope=dqr, **kw)
        accs.append(acc)
    acc = torch.stack(accs).sum(0)
    dk, dv, dkr = S.sfa_dkv_finalize(acc, dp.q, dp.k, dp.qr, dp.idx, layout=p.layout, deterministic=True,
                                     dout_absmax=dmax, scale=p.scale, actual_seq_lengths_q=dp.sq)
    got = (dq, dk, dv, dqr, dkr)
    for name, g, f in zip(("dQuery", "dKey", "dValue", "dQueryRope", "dKeyRope"), got, full):
        assert torch.equal(g, f), f"{case}: {name} differs from sfa_grad"
    compare_grads(grads_np(got, p), oracle_backward(p, out, m, l), what=f"rows {case}/")


def test_host_pipeline_small_gradient():
    """sfa_grad_host in deterministic mode (dOut copied first, its max setting the grid) at
    dOut x 1e-8: bit-identical to sfa_grad."""
    import sparse_attention_backward_sfa_b200 as S
    p = scaled_problem("fused_n128", 1e-8, seed=923)
    dp = DevProblem(p)
    prepare_oracle_forward(p, dp)
    full = dp.grad_gpu(deterministic=True)
    h = lambda x: None if x is None else x.cpu().pin_memory()
    got = S.sfa_grad_host(h(dp.q), h(dp.k), True, h(dp.idx), h(dp.do), h(dp.out), h(dp.smax), h(dp.ssum),
                          h(dp.qr), h(dp.kr), scale=p.scale, sparse_block_size=p.block_size, layout=p.layout,
                          sparse_mode=p.sparse_mode, deterministic=True, actual_seq_lengths_q=h(dp.sq),
                          actual_seq_lengths_kv=h(dp.skv), chunks=3)
    for name, g, f in zip(("dQuery", "dKey", "dValue", "dQueryRope", "dKeyRope"), got, full):
        assert torch.equal(g, f.cpu()), f"{name} differs from sfa_grad"
