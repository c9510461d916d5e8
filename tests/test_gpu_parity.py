"""GPU parity of the library against the CPU oracle (same seeded inputs).

Integer work (index compaction) is compared bit for bit; bf16 outputs with
max|err| <= 2e-2*max|ref| and cosine >= 0.9999 per tensor; deterministic mode
bit for bit run to run."""
import numpy as np
import pytest
import torch

from oracle import sfa_oracle as O
from workloads import make_fa_problem, make_problem, tiny_problem
from parity import (DevFA, DevProblem, assert_close, compare_grads, grads_np, oracle_backward, oracle_forward,
                    prepare_oracle_forward)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_backward_sfa_b200 import build
    build.build()


def tiny(seed, **kw):
    base = dict(D=512, Dr=64)
    base.update(kw)
    return tiny_problem(seed, **base)


CASES = {
    "bsnd_mode0_bs1": dict(layout="BSND", B=2, S1=9, S2=70, N1=2, topk=24, block_size=1, sparse_mode=0),
    "bsnd_mode3_bs4_messy": dict(layout="BSND", B=2, S1=12, S2=40, N1=4, topk=9, block_size=4, sparse_mode=3,
                                 index_mode="messy", seqlens_q=[12, 7], seqlens_kv=[40, 23]),
    "tnd_mode3_bs16_causal": dict(layout="TND", seqlens_q=[33, 1, 20], seqlens_kv=[33, 5, 47], N1=2, topk=5,
                                  block_size=16, sparse_mode=3, index_mode="causal"),
    "tnd_mode0_bs3_dup": dict(layout="TND", seqlens_q=[5, 6], seqlens_kv=[17, 9], N1=1, topk=8, block_size=3,
                              sparse_mode=0, index_mode="messy"),
    "bsnd_q_longer_than_kv": dict(layout="BSND", B=1, S1=20, S2=8, N1=2, topk=8, block_size=1, sparse_mode=3,
                                  index_mode="messy"),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_compact_indices_bit_exact(case):
    import sparse_attention_backward_sfa_b200 as S
    p = tiny(7, **CASES[case])
    dp = DevProblem(p)
    blocks, nb, nr = S.compact_indices(dp.idx, dp.k, dp.q, dp.qr, sparse_block_size=p.block_size, layout=p.layout,
                                       sparse_mode=p.sparse_mode, actual_seq_lengths_q=dp.sq,
                                       actual_seq_lengths_kv=dp.skv)
    blocks, nb, nr = blocks.cpu().numpy(), nb.cpu().numpy(), nr.cpu().numpy()
    spans = O.make_spans(p.layout, p.B, p.S1, p.S2, p.seqlens_q, p.seqlens_kv)
    seen = set()
    for sp in spans:
        for pos in range(sp.q_len):
            t = sp.q_start + pos
            seen.add(t)
            ref_rows = O.selected_rows(p.indices[t], p.block_size, pos, sp.q_len, sp.kv_len, p.sparse_mode)
            got_rows = []
            for b in blocks[t, :nb[t]].tolist():
                for j in range(b * p.block_size, b * p.block_size + p.block_size):
                    if j < sp.kv_len and (p.sparse_mode == 0 or j <= pos + sp.kv_len - sp.q_len):
                        got_rows.append(j)
            assert got_rows == ref_rows, (t, got_rows, ref_rows)
            assert nr[t] == len(ref_rows)
    for t in range(p.T1):
        if t not in seen:
            assert nb[t] == 0 and nr[t] == 0


KEY_ROW_CASES = {
    "bsnd_bs5_messy": dict(layout="BSND", B=2, S1=11, S2=83, N1=1, topk=14, block_size=5, sparse_mode=3,
                           index_mode="messy", seqlens_q=[11, 6], seqlens_kv=[83, 40]),
    "tnd_bs16_messy": dict(layout="TND", seqlens_q=[21, 3, 30], seqlens_kv=[70, 9, 130], N1=1, topk=12,
                           block_size=16, sparse_mode=3, index_mode="messy"),
    "tnd_bs32_messy_mode0": dict(layout="TND", seqlens_q=[9, 17], seqlens_kv=[100, 250], N1=1, topk=10,
                                 block_size=32, sparse_mode=0, index_mode="messy"),
    "bsnd_bs16_q_longer": dict(layout="BSND", B=1, S1=40, S2=35, N1=1, topk=6, block_size=16, sparse_mode=3,
                               index_mode="messy"),
}


@pytest.mark.parametrize("case", sorted(KEY_ROW_CASES))
@pytest.mark.parametrize("sorted_blocks", [False, True])
@pytest.mark.parametrize("block_aligned", [False, True])
def test_key_rows_bit_exact(case, sorted_blocks, block_aligned):
    """The expanded key-row lists the fused kernels read (after the optional block sort, with the
    block-aligned padding slots) against the oracle's selected rows: exact rows in index order
    (unsorted), the same multiset (sorted), every padding slot flagged and every kept block whole."""
    import sparse_attention_backward_sfa_b200 as S
    p = tiny(29, **KEY_ROW_CASES[case])
    dp = DevProblem(p)
    bs = p.block_size
    blocks, nb, rows, cnt = S.key_rows(dp.idx, dp.k, dp.q, dp.qr, sparse_block_size=bs, layout=p.layout,
                                       sparse_mode=p.sparse_mode, sorted_blocks=sorted_blocks,
                                       block_aligned=block_aligned, actual_seq_lengths_q=dp.sq,
                                       actual_seq_lengths_kv=dp.skv)
    blocks, nb, rows, cnt = (x.cpu().numpy() for x in (blocks, nb, rows, cnt))
    flag = np.int64(1) << 31
    seen = set()
    for sp in O.make_spans(p.layout, p.B, p.S1, p.S2, p.seqlens_q, p.seqlens_kv):
        for pos in range(sp.q_len):
            t = sp.q_start + pos
            seen.add(t)
            ref = [sp.kv_start + j for j in O.selected_rows(p.indices[t], bs, pos, sp.q_len, sp.kv_len,
                                                             p.sparse_mode)]
            kept = blocks[t, :nb[t]].astype(np.int64)
            if sorted_blocks:
                assert (np.diff(kept) >= 0).all(), (t, kept)
            got = rows[t, :cnt[t]].astype(np.int64) & 0xFFFFFFFF
            if block_aligned:
                assert cnt[t] == nb[t] * bs
                valid = got[(got & flag) == 0]
                for i, b in enumerate(kept.tolist()):  # every kept block whole, its cut rows flagged
                    grp = got[i * bs:(i + 1) * bs]
                    first = sp.kv_start + b * bs
                    np.testing.assert_array_equal(grp & ~flag, np.arange(first, first + bs))
                    keep = [j for j in range(b * bs, b * bs + bs) if j < sp.kv_len and
                            (p.sparse_mode == 0 or j <= pos + sp.kv_len - sp.q_len)]
                    np.testing.assert_array_equal((grp & flag) == 0, np.arange(bs) < len(keep))
            else:
                valid = got
                assert cnt[t] == len(ref)
            if sorted_blocks:
                assert sorted(valid.tolist()) == sorted(ref), (t,)
            else:
                assert valid.tolist() == ref, (t, valid.tolist(), ref)
    for t in range(p.T1):
        if t not in seen:
            assert nb[t] == 0 and cnt[t] == 0


def test_softmax_grad_rowsum():
    import sparse_attention_backward_sfa_b200 as S
    p = tiny(3, layout="BSND", B=1, S1=37, S2=16, N1=4, topk=4)
    dp = DevProblem(p)
    out = np.asarray(np.random.default_rng(1).standard_normal((p.T1, p.N1, p.D)), np.float32)
    dp.set_forward(out, np.zeros((p.T1, p.N1)), np.ones((p.T1, p.N1)))
    got = S.softmax_grad_rowsum(dp.do, dp.out, dp.k, dp.qr, dp.idx, layout=p.layout).cpu().numpy()
    o16 = dp.out.float().cpu().numpy().reshape(p.T1, p.N1, p.D).astype(np.float64)
    ref = (p.dout.astype(np.float64) * o16).sum(-1)
    np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-4)


@pytest.mark.parametrize("case", sorted(CASES))
def test_sfa_fwd_parity(case):
    p = tiny(11, **CASES[case])
    dp = DevProblem(p)
    out, m, l = dp.forward_gpu()
    ro, rm, rl = oracle_forward(p)
    go, gm, gl = dp.host_fwd_inputs()
    assert_close("out", go, ro)
    np.testing.assert_allclose(gm, rm, rtol=2e-5, atol=2e-5)
    np.testing.assert_allclose(gl, rl, rtol=2e-5, atol=1e-6)


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("det", [False, True])
def test_sfa_grad_generic_parity(case, det):
    p = tiny(13, **CASES[case])
    dp = DevProblem(p)
    out, m, l = prepare_oracle_forward(p, dp)
    got = grads_np(dp.grad_gpu(deterministic=det), p)
    ref = oracle_backward(p, out, m, l)
    compare_grads(got, ref, what=f"{case}/det={det}/")


def test_sfa_grad_value_distinct_from_key():
    p = tiny(17, layout="BSND", B=1, S1=6, S2=30, N1=2, topk=10, block_size=2, sparse_mode=3, index_mode="causal",
             value_is_key=False)
    dp = DevProblem(p)
    out, m, l = prepare_oracle_forward(p, dp)
    compare_grads(grads_np(dp.grad_gpu(), p), oracle_backward(p, out, m, l), what="value!=key/")


def test_sfa_grad_fp16():
    p = tiny(19, layout="TND", seqlens_q=[8, 5], seqlens_kv=[20, 9], N1=2, topk=6, block_size=2, sparse_mode=3,
             index_mode="causal")
    dp = DevProblem(p, dtype=torch.float16)
    # fp16 inputs: round the fp32 values through fp16 for the oracle too
    for a in (p.q, p.q_rope, p.k, p.k_rope, p.dout):
        a[...] = a.astype(np.float16).astype(np.float32)
    dp = DevProblem(p, dtype=torch.float16)
    out, m, l = prepare_oracle_forward(p, dp)
    compare_grads(grads_np(dp.grad_gpu(), p), oracle_backward(p, out, m, l), what="fp16/")


def test_sfa_rows_without_keys_and_padding_tokens():
    """All -1 rows, blocks past S2_b, BSND padding tokens: zero dQuery rows."""
    p = tiny(23, layout="BSND", B=2, S1=6, S2=12, N1=2, topk=4, block_size=4, sparse_mode=0,
             seqlens_q=[4, 6], seqlens_kv=[12, 5])
    p.indices[0, :] = -1
    p.indices[1, :] = [7, 9, -3, 100]
    dp = DevProblem(p)
    out, m, l = prepare_oracle_forward(p, dp)
    got = grads_np(dp.grad_gpu(), p)
    compare_grads(got, oracle_backward(p, out, m, l), what="empty/")
    assert not got[0][0].any() and not got[0][1].any()
    assert not got[0][4:6].any()  # padding rows of batch 0


@pytest.mark.parametrize("det", [False, True])
def test_workload1_full(det):
    p = make_problem(1)
    dp = DevProblem(p)
    out, m, l = prepare_oracle_forward(p, dp)
    got = grads_np(dp.grad_gpu(deterministic=det), p)
    compare_grads(got, oracle_backward(p, out, m, l), what="cfg1/")


def test_deterministic_bit_identical_generic():
    p = tiny(29, layout="TND", seqlens_q=[40, 24], seqlens_kv=[40, 64], N1=4, topk=12, block_size=4,
             sparse_mode=3, index_mode="causal")
    dp = DevProblem(p)
    prepare_oracle_forward(p, dp)
    a = [r.clone() for r in dp.grad_gpu(deterministic=True)]
    for _ in range(2):
        b = dp.grad_gpu(deterministic=True)
        for x, y in zip(a, b):
            assert torch.equal(x.view(torch.int16), y.view(torch.int16))


# ---------------------------------------------------------------------------
# Dense varlen FA
# ---------------------------------------------------------------------------
def _fa_case(fp, det=False):
    d = DevFA(fp)
    d.forward_gpu()
    out = d.out.float().cpu().numpy()
    sm = d.smax.cpu().numpy().astype(np.float64)
    ss = d.ssum.cpu().numpy().astype(np.float64)
    ro, rm, rl = O.fa_forward(fp.q, fp.k, fp.v, fp.cu_seqlens_q, fp.cu_seqlens_kv, fp.scale, fp.sparse_mode)
    assert_close("fa out", out, ro)
    np.testing.assert_allclose(sm, rm, rtol=2e-5, atol=2e-5)
    np.testing.assert_allclose(ss, rl, rtol=2e-5, atol=1e-6)
    dq, dk, dv = (x.float().cpu().numpy() for x in d.grad_gpu(deterministic=det))
    rq, rk, rv = O.fa_backward(fp.q, fp.k, fp.v, fp.dy, sm, ss, out, fp.cu_seqlens_q, fp.cu_seqlens_kv, fp.scale,
                               fp.sparse_mode)
    assert_close("fa dq", dq, rq)
    assert_close("fa dk", dk, rk)
    assert_close("fa dv", dv, rv)


@pytest.mark.parametrize("det", [False, True])
def test_fa_small_gqa_bottom_right(det):
    _fa_case(make_fa_problem(seed=5, lens=(37, 1, 64), N=8, Nkv=2, D=128, sparse_mode=3, kv_lens=(50, 9, 64)), det)


def test_fa_small_mode0_d64():
    _fa_case(make_fa_problem(seed=6, lens=(20, 45), N=4, Nkv=4, D=64, sparse_mode=0))


@pytest.mark.parametrize("det", [False, True])
def test_fa_d64_gqa_bottom_right(det):
    """Head dim 64 on the tensor-core kernel: GQA, several 128-key blocks with ragged tails,
    sequences with fewer queries than keys (bottom-right causal), an empty query span."""
    _fa_case(make_fa_problem(seed=8, lens=(150, 0, 77, 300), N=8, Nkv=2, D=64, sparse_mode=3,
                             kv_lens=(200, 30, 77, 300)), det)


def test_fa_d64_workload2_shape():
    """Workload 2's sequences and heads at head dim 64."""
    _fa_case(make_fa_problem(seed=9, D=64))


def test_fa_d64_fp16():
    import sparse_attention_backward_sfa_b200 as S
    fp = make_fa_problem(seed=10, lens=(64, 190), N=4, Nkv=1, D=64, sparse_mode=3)
    d = DevFA(fp, dtype=torch.float16)
    d.forward_gpu()
    out = d.out.float().cpu().numpy()
    sm = d.smax.cpu().numpy().astype(np.float64)
    ss = d.ssum.cpu().numpy().astype(np.float64)
    dq, dk, dv = (x.float().cpu().numpy() for x in d.grad_gpu())
    rq, rk, rv = O.fa_backward(fp.q, fp.k, fp.v, fp.dy, sm, ss, out, fp.cu_seqlens_q, fp.cu_seqlens_kv, fp.scale,
                               fp.sparse_mode)
    assert_close("fa16 dq", dq, rq)
    assert_close("fa16 dk", dk, rk)
    assert_close("fa16 dv", dv, rv)


def test_fa_workload2_full():
    _fa_case(make_fa_problem())


ODD_N1 = {
    # the N1 values the page lists for Ascend 950 (3/6/12/24/48), served by the CUDA-core kernel
    "n3_bsnd_bs1": dict(layout="BSND", B=2, S1=13, S2=90, N1=3, topk=40, block_size=1, sparse_mode=3,
                        index_mode="causal", seqlens_q=[13, 8], seqlens_kv=[90, 51]),
    "n6_tnd_bs16": dict(layout="TND", seqlens_q=[40, 7], seqlens_kv=[60, 100], N1=6, topk=6, block_size=16,
                        sparse_mode=3, index_mode="causal"),
    "n12_tnd_bs1": dict(layout="TND", seqlens_q=[19, 30], seqlens_kv=[19, 64], N1=12, topk=48, block_size=1,
                        sparse_mode=3, index_mode="messy"),
    "n24_bsnd_bs16": dict(layout="BSND", B=1, S1=21, S2=130, N1=24, topk=9, block_size=16, sparse_mode=3,
                          index_mode="causal"),
    "n48_tnd_bs16": dict(layout="TND", seqlens_q=[17, 5], seqlens_kv=[80, 33], N1=48, topk=6, block_size=16,
                         sparse_mode=3, index_mode="causal"),
    "n48_bsnd_bs1": dict(layout="BSND", B=1, S1=9, S2=64, N1=48, topk=32, block_size=1, sparse_mode=3,
                         index_mode="causal"),
}


@pytest.mark.parametrize("case", sorted(ODD_N1))
@pytest.mark.parametrize("det", [False, True])
def test_odd_n1_parity(case, det):
    p = tiny(41, **ODD_N1[case])
    dp = DevProblem(p)
    out, m, l = prepare_oracle_forward(p, dp)
    got = grads_np(dp.grad_gpu(deterministic=det), p)
    compare_grads(got, oracle_backward(p, out, m, l), what=f"{case}/det={det}/")


@pytest.mark.parametrize("case", ["n6_tnd_bs16", "n48_bsnd_bs1"])
def test_odd_n1_forward_parity(case):
    p = tiny(43, **ODD_N1[case])
    dp = DevProblem(p)
    out, m, l = (x.float().cpu().numpy() for x in dp.forward_gpu())
    ro, rm, rl = oracle_forward(p)
    assert_close(f"{case} out", out.reshape(ro.shape), ro)
    np.testing.assert_allclose(m.reshape(rm.shape), rm, rtol=1e-4, atol=1e-4)
    np.testing.assert_allclose(l.reshape(rl.shape), rl, rtol=1e-4, atol=1e-6)


@pytest.mark.parametrize("D", [192, 256])
@pytest.mark.parametrize("det", [False, True])
def test_fa_large_head_dims_gqa(D, det):
    _fa_case(make_fa_problem(seed=7 + D, lens=(29, 50), N=6, Nkv=2, D=D, sparse_mode=3, kv_lens=(41, 50)), det)


def test_fa_page2_worked_example():
    """All-ones TND T=256, N=1, D=128, stats 3.0/3.0, scale 0.088388, mode 0:
    dq = dk = 0 exactly, dv = 256*exp(128*0.088388 - 3)/3 (bf16-rounded)."""
    import math
    import sparse_attention_backward_sfa_b200 as S
    T, D = 256, 128
    one = torch.ones(T, 1, D, dtype=torch.bfloat16, device="cuda")
    st = torch.full((T, 1, 8), 3.0, device="cuda")
    dq, dk, dv = S.fa_grad(one, one, one, one, st, st, one, [256], [256], scale=0.088388, sparse_mode=0)
    assert not dq.float().any() and not dk.float().any()
    ref = T * math.exp(D * 0.088388 - 3.0) / 3.0
    assert abs(dv.float().max().item() - ref) <= 2 ** -7 * ref and abs(dv.float().min().item() - ref) <= 2 ** -7 * ref
