"""GPU parity of the paired-row backward (N1 = 128, value == key): adjacent query rows whose
kept block lists are identical run on the two CTAs of a cluster and share every key tile's
dK~ / dV reduction (SparseFlashAttentionGrad README, 功能说明: a key's gradient sums over
every row that selected it).  Cases cover contiguous tiles (every causal block selected) and
gathered ones (the same random blocks for both rows of a pair), block sizes 16 and 32, both
layouts, fp16, rows left unpaired (odd counts, lists that differ), row ranges that start on
an odd row, and deterministic bit identity."""
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


def tiny(seed, **kw):
    base = dict(D=512, Dr=64, N1=128)
    base.update(kw)
    return tiny_problem(seed, **base)


def pair_rows(p, rng_seed=0):
    """Give every odd row the indices of the row before it (same sequence), as a shuffled copy:
    the pair then shares its blocks, and the kernel sees them in sorted order."""
    rng = np.random.default_rng(rng_seed)
    idx = p.indices.copy()
    for t in range(1, idx.shape[0], 2):
        row = idx[t - 1].copy()
        rng.shuffle(row)
        idx[t] = row
    p.indices = idx
    return p


CASES = {
    # every causal block: contiguous 128-key tiles, ragged tails, two sequences (pairs within each)
    "tnd_bs16_all_blocks": dict(layout="TND", seqlens_q=[260, 46], seqlens_kv=[260, 301], topk=40, block_size=16,
                                sparse_mode=3, index_mode="causal"),
    # block size 32 (a tile holds four blocks), BSND with two batches, varlen
    "bsnd_bs32_all_blocks": dict(layout="BSND", B=2, S1=96, S2=200, topk=16, block_size=32, sparse_mode=3,
                                 index_mode="causal", seqlens_q=[96, 64], seqlens_kv=[200, 130]),
    # an odd number of rows in the first sequence: its last row is unpaired, the second sequence
    # then starts on an odd row, so its rows pair across the sequence boundary test (not paired)
    "tnd_odd_lengths": dict(layout="TND", seqlens_q=[131, 64], seqlens_kv=[131, 64], topk=12, block_size=16,
                            sparse_mode=3, index_mode="causal"),
}


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("det", [False, True])
def test_pair_parity(case, det):
    p = tiny(1201, **CASES[case])
    dp = DevProblem(p)
    out, m, l = prepare_oracle_forward(p, dp)
    got = grads_np(dp.grad_gpu(deterministic=det), p)
    compare_grads(got, oracle_backward(p, out, m, l), what=f"{case}/det={det}/")


@pytest.mark.parametrize("det", [False, True])
def test_pair_gathered_tiles(det):
    """Random (non-contiguous) blocks shared by each pair: key tiles by tile::gather4, mode 0."""
    p = pair_rows(tiny(1203, layout="BSND", B=1, S1=12, S2=700, topk=30, block_size=16, sparse_mode=0,
                       index_mode="distinct"))
    dp = DevProblem(p)
    out, m, l = prepare_oracle_forward(p, dp)
    got = grads_np(dp.grad_gpu(deterministic=det), p)
    compare_grads(got, oracle_backward(p, out, m, l), what=f"gathered/det={det}/")


def test_pair_gathered_block_size_one():
    """Block size 1: the pair's rows select the same random key rows (the same order)."""
    p = tiny(1205, layout="TND", seqlens_q=[10], seqlens_kv=[500], topk=260, block_size=1, sparse_mode=0,
             index_mode="distinct")
    idx = p.indices.copy()
    idx[1::2] = idx[0::2]
    p.indices = idx
    dp = DevProblem(p)
    out, m, l = prepare_oracle_forward(p, dp)
    got = grads_np(dp.grad_gpu(deterministic=True), p)
    compare_grads(got, oracle_backward(p, out, m, l), what="bs1 pairs/")


def test_pair_fp16():
    p = tiny(1207, **CASES["tnd_bs16_all_blocks"])
    dp = DevProblem(p, dtype=torch.float16)
    from parity import oracle_forward
    o, m, l = oracle_forward(p)
    out_q = np.asarray(o, np.float16).astype(np.float32)
    dp.set_forward(out_q, np.asarray(m, np.float32), np.asarray(l, np.float32))
    got = grads_np(dp.grad_gpu(deterministic=False), p)
    ref = oracle_backward(p, out_q.astype(np.float64), np.asarray(m, np.float32).astype(np.float64),
                          np.asarray(l, np.float32).astype(np.float64))
    compare_grads(got, ref, what="fp16 pairs/")


def test_pair_deterministic_bit_identical():
    p = pair_rows(tiny(1209, **CASES["tnd_bs16_all_blocks"]))
    dp = DevProblem(p)
    prepare_oracle_forward(p, dp)
    a = [r.clone() for r in dp.grad_gpu(deterministic=True)]
    for _ in range(2):
        b = dp.grad_gpu(deterministic=True)
        for x, y in zip(a, b):
            assert torch.equal(x.view(torch.int16), y.view(torch.int16))


@pytest.mark.parametrize("det", [False, True])
def test_pair_row_ranges_from_odd_rows(det):
    """Row ranges starting on odd rows pair differently than the whole call; the summed
    accumulators still match the oracle (and, deterministic, each other run to run)."""
    import sparse_attention_backward_sfa_b200 as S
    p = tiny(1211, **CASES["tnd_bs16_all_blocks"])
    dp = DevProblem(p)
    out, m, l = prepare_oracle_forward(p, dp)
    kw = dp.kw()
    ranges = [(0, 37), (37, 170), (170, p.T1)]
    dmax = None
    if det:
        dmax = torch.zeros(1, dtype=torch.float32, device="cuda")
        S.dout_absmax(dp.do, dp.q, dp.k, dp.qr, dp.idx, layout=p.layout, actual_seq_lengths_q=dp.sq, into=dmax)
    acc = S.sfa_dkv_accumulator(dp.q, dp.k, dp.qr, dp.idx, layout=p.layout, deterministic=det,
                                actual_seq_lengths_q=dp.sq)
    dq = torch.zeros_like(dp.q)
    dqr = torch.zeros_like(dp.qr)
    for rb, re_ in ranges:
        S.sfa_grad_rows(dp.q, dp.k, dp.v, dp.idx, dp.do, dp.out, dp.smax, dp.ssum, dp.qr, dp.kr, row_begin=rb,
                        row_end=re_, dkv_accum=acc, deterministic=det, dout_absmax=dmax, d_query=dq,
                        d_query_rope=dqr, **kw)
    dk, dv, dkr = S.sfa_dkv_finalize(acc, dp.q, dp.k, dp.qr, dp.idx, layout=p.layout, deterministic=det,
                                     dout_absmax=dmax, scale=p.scale, actual_seq_lengths_q=dp.sq)
    compare_grads(grads_np((dq, dk, dv, dqr, dkr), p), oracle_backward(p, out, m, l), what=f"ranges/det={det}/")
