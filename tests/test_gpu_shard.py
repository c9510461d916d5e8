"""GPU checks of the query-row sharded backward (sfa_grad_rows + sfa_dkv_finalize):
the key-side accumulators of disjoint row ranges add up to sfa_grad's result —
bit-identical in deterministic mode (64-bit fixed point) — and the dQuery rows of
each range are the ones sfa_grad writes.  The ranges run one after another on one
GPU; several GPUs would sum the same accumulators with an all-reduce."""
import numpy as np
import pytest
import torch

from workloads import tiny_problem
from parity import DevProblem, compare_grads, grads_np, oracle_backward, prepare_oracle_forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_backward_sfa_b200 import build
    build.build()


CASES = {
    # CUDA-core path (N1 < 64)
    "generic_n2_bsnd": dict(layout="BSND", B=2, S1=7, S2=90, N1=2, topk=30, block_size=1, sparse_mode=3,
                            index_mode="causal"),
    # fused tensor-core path, several tiles per row, block indices
    "fused_n128_tnd_bs16": dict(layout="TND", seqlens_q=[70, 3, 150], seqlens_kv=[70, 260, 150], N1=128, topk=12,
                                block_size=16, sparse_mode=3, index_mode="causal"),
    "fused_n64_bsnd": dict(layout="BSND", B=1, S1=11, S2=400, N1=64, topk=300, block_size=1, sparse_mode=0),
}


def sharded(dp, ranges, det, separate=False):
    """sfa_grad_rows over `ranges`; one shared accumulator, or one per range summed afterwards."""
    import sparse_attention_backward_sfa_b200 as S
    kw = dp.kw()
    mk = lambda: S.sfa_dkv_accumulator(dp.q, dp.k, dp.qr, dp.idx, layout=kw["layout"], deterministic=det,
                                       actual_seq_lengths_q=dp.sq)
    acc = mk()
    accs = []
    dq = torch.zeros_like(dp.q)
    dqr = torch.zeros_like(dp.qr)
    dmax = None
    if det:
        # each range's max|dOut| max-merged: what the ranks' max all-reduce computes
        dmax = torch.zeros(1, dtype=torch.float32, device=dp.q.device)
        for rb, re_ in ranges:
            S.dout_absmax(dp.do, dp.q, dp.k, dp.qr, dp.idx, layout=kw["layout"], row_begin=rb, row_end=re_,
                          actual_seq_lengths_q=dp.sq, into=dmax)
    for rb, re_ in ranges:
        a = mk() if separate else acc
        S.sfa_grad_rows(dp.q, dp.k, dp.v, dp.idx, dp.do, dp.out, dp.smax, dp.ssum, dp.qr, dp.kr, row_begin=rb,
                        row_end=re_, dkv_accum=a, deterministic=det, dout_absmax=dmax, d_query=dq,
                        d_query_rope=dqr, **kw)
        accs.append(a)
    if separate:
        acc = torch.stack(accs).sum(0)  # what an all-reduce of the ranks' accumulators computes
    dk, dv, dkr = S.sfa_dkv_finalize(acc, dp.q, dp.k, dp.qr, dp.idx, layout=kw["layout"], deterministic=det,
                                     dout_absmax=dmax, scale=kw["scale"], actual_seq_lengths_q=dp.sq)
    return dq, dk, dv, dqr, dkr


def three_ranges(T1):
    """Three ranges with boundaries on even rows (pairs of rows stay together, as in the whole call)."""
    a, b = 2 * (T1 // 6), 2 * (T1 // 3) + 2
    b = min(b, T1)
    return [(0, a), (a, b), (b, T1)]


@pytest.mark.parametrize("case", sorted(CASES))
def test_sharded_deterministic_is_bit_identical(case):
    p = tiny_problem(311, D=512, Dr=64, **CASES[case])
    dp = DevProblem(p)
    prepare_oracle_forward(p, dp)
    full = dp.grad_gpu(deterministic=True)
    for separate in (False, True):
        got = sharded(dp, three_ranges(p.T1), True, separate=separate)
        for name, g, f in zip(("dQuery", "dKey", "dValue", "dQueryRope", "dKeyRope"), got, full):
            assert torch.equal(g, f), f"{case}: {name} differs from sfa_grad (separate={separate})"


@pytest.mark.parametrize("case", sorted(CASES))
def test_sharded_atomic_matches_oracle(case):
    p = tiny_problem(313, D=512, Dr=64, **CASES[case])
    dp = DevProblem(p)
    out, m, l = prepare_oracle_forward(p, dp)
    got = grads_np(sharded(dp, three_ranges(p.T1), False, separate=True), p)
    compare_grads(got, oracle_backward(p, out, m, l), what=f"sharded {case}/")


def test_rows_outside_range_untouched_and_range_checked():
    import sparse_attention_backward_sfa_b200 as S
    p = tiny_problem(317, D=512, Dr=64, **CASES["fused_n64_bsnd"])
    dp = DevProblem(p)
    prepare_oracle_forward(p, dp)
    kw = dp.kw()
    acc = S.sfa_dkv_accumulator(dp.q, dp.k, dp.qr, dp.idx, layout=kw["layout"], deterministic=False)
    dq = torch.full_like(dp.q, 7.0)
    dqr = torch.full_like(dp.qr, 7.0)
    S.sfa_grad_rows(dp.q, dp.k, dp.v, dp.idx, dp.do, dp.out, dp.smax, dp.ssum, dp.qr, dp.kr, row_begin=3, row_end=5,
                    dkv_accum=acc, d_query=dq, d_query_rope=dqr, **kw)
    flat = dq.reshape(p.T1, -1)
    assert bool((flat[:3] == 7).all()) and bool((flat[5:] == 7).all())
    assert not bool((flat[3:5] == 7).all())
    with pytest.raises(S.SfaError):
        S.sfa_grad_rows(dp.q, dp.k, dp.v, dp.idx, dp.do, dp.out, dp.smax, dp.ssum, dp.qr, dp.kr, row_begin=2,
                        row_end=p.T1 + 1, dkv_accum=acc, d_query=dq, d_query_rope=dqr, **kw)


@pytest.mark.parametrize("case", sorted(CASES))
def test_rows_range_reads_only_its_rows(case):
    """A row range reads only its own rows of the indices and of the query-side inputs (the host
    pipeline copies them chunk by chunk): with every other row poisoned (NaN inputs, scrambled
    indices) the range's dQuery rows and key-side sums are bit-identical to the clean call's."""
    import sparse_attention_backward_sfa_b200 as S
    p = tiny_problem(319, D=512, Dr=64, **CASES[case])
    dp = DevProblem(p)
    prepare_oracle_forward(p, dp)
    kw = dp.kw()
    T1 = p.T1
    a, b = 2 * (T1 // 4), min(T1, 2 * (T1 // 4) + 4)

    def run(q, qr, do, out, smax, ssum, idx):
        acc = S.sfa_dkv_accumulator(q, dp.k, qr, idx, layout=kw["layout"], deterministic=True,
                                    actual_seq_lengths_q=dp.sq)
        dmax = torch.zeros(1, dtype=torch.float32, device=q.device)
        S.dout_absmax(do, q, dp.k, qr, idx, layout=kw["layout"], row_begin=a, row_end=b,
                      actual_seq_lengths_q=dp.sq, into=dmax)
        dq, dqr = torch.zeros_like(q), torch.zeros_like(qr)
        S.sfa_grad_rows(q, dp.k, dp.v, idx, do, out, smax, ssum, qr, dp.kr, row_begin=a, row_end=b, dkv_accum=acc,
                        deterministic=True, dout_absmax=dmax, d_query=dq, d_query_rope=dqr, **kw)
        torch.cuda.synchronize()
        return dq.reshape(T1, -1)[a:b], dqr.reshape(T1, -1)[a:b], acc

    clean = run(dp.q, dp.qr, dp.do, dp.out, dp.smax, dp.ssum, dp.idx)
    g = torch.Generator(device="cpu").manual_seed(5)

    def poison(x):
        y = x.clone()
        flat = y.reshape(T1, -1)
        keep = flat[a:b].clone()
        if y.dtype == torch.int32:
            flat.copy_(torch.randint(-1, 1 << 20, flat.shape, generator=g, dtype=torch.int32).to(y.device))
        else:
            flat.fill_(float("nan"))
        flat[a:b] = keep
        return y

    got = run(*(poison(x) for x in (dp.q, dp.qr, dp.do, dp.out, dp.smax, dp.ssum, dp.idx)))
    for name, x, y in zip(("dQuery rows", "dQueryRope rows", "key-side accumulator"), got, clean):
        assert torch.equal(x, y), f"{case}: {name} depend on rows outside the range"


def test_balanced_split_of_real_counts():
    """The bench's work split on a causal problem: contiguous, covering, boundaries on even rows
    (row pairs stay together) and balanced within three rows."""
    import sparse_attention_backward_sfa_b200 as S
    p = tiny_problem(319, D=512, Dr=64, **CASES["fused_n128_tnd_bs16"])
    dp = DevProblem(p)
    _, _, nr = S.compact_indices(dp.idx, dp.k, dp.q, dp.qr, sparse_block_size=p.block_size, layout=p.layout,
                                 sparse_mode=p.sparse_mode, actual_seq_lengths_q=dp.sq, actual_seq_lengths_kv=dp.skv)
    w = nr.cpu().numpy().astype(np.float64)
    for parts in (2, 3, 8):
        r = S.balanced_row_ranges(w, parts)
        assert r[0][0] == 0 and r[-1][1] == p.T1 and all(r[i][1] == r[i + 1][0] for i in range(parts - 1))
        assert all(b % 2 == 0 for _, b in r[:-1])
        sums = [w[a:b].sum() for a, b in r]
        assert max(sums) - w.sum() / parts <= 3 * w.max() + 1e-9


@pytest.mark.parametrize("case", ["generic_n2_bsnd", "fused_n128_tnd_bs16"])
def test_host_pipeline_matches_sfa_grad(case):
    """sfa_grad_host (pinned host tensors, chunked rows, copies overlapped) gives sfa_grad's
    results: bit-identical in deterministic mode."""
    import sparse_attention_backward_sfa_b200 as S
    p = tiny_problem(331, D=512, Dr=64, **CASES[case])
    dp = DevProblem(p)
    prepare_oracle_forward(p, dp)
    full = dp.grad_gpu(deterministic=True)
    h = lambda x: None if x is None else x.cpu().pin_memory()
    pl = S.HostPipeline(torch.device("cuda"))
    for chunks in (1, 3):
        got = S.sfa_grad_host(h(dp.q), h(dp.k), True, h(dp.idx), h(dp.do), h(dp.out), h(dp.smax), h(dp.ssum),
                              h(dp.qr), h(dp.kr), scale=p.scale, sparse_block_size=p.block_size, layout=p.layout,
                              sparse_mode=p.sparse_mode, deterministic=True, actual_seq_lengths_q=h(dp.sq),
                              actual_seq_lengths_kv=h(dp.skv), chunks=chunks, pipeline=pl)
        for name, g, f in zip(("dQuery", "dKey", "dValue", "dQueryRope", "dKeyRope"), got, full):
            assert torch.equal(g, f.cpu()), f"{case}: {name} differs (chunks={chunks})"
