"""GPU parity of the fused tcgen05 backward (N1 in {64, 128}, value == key)
against the CPU oracle: several key tiles with a ragged tail, both layouts,
block sizes 1 / 5 / 16, sparse modes 0 / 3, messy indices, fp16, determinism."""
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
    base = dict(D=512, Dr=64)
    base.update(kw)
    return tiny_problem(seed, **base)


FUSED = {
    "n128_bsnd_mode0_bs1_3tiles": dict(layout="BSND", B=1, S1=5, S2=700, N1=128, topk=300, block_size=1,
                                       sparse_mode=0),
    "n64_bsnd_mode3_varlen": dict(layout="BSND", B=2, S1=40, S2=300, N1=64, topk=200, block_size=1, sparse_mode=3,
                                  index_mode="causal", seqlens_q=[40, 17], seqlens_kv=[300, 140]),
    "n128_tnd_bs16_causal": dict(layout="TND", seqlens_q=[70, 3, 150], seqlens_kv=[70, 260, 150], N1=128, topk=12,
                                 block_size=16, sparse_mode=3, index_mode="causal"),
    "n64_tnd_messy_bs5": dict(layout="TND", seqlens_q=[9, 12], seqlens_kv=[333, 90], N1=64, topk=40, block_size=5,
                              sparse_mode=0, index_mode="messy"),
    "n128_exact_tile": dict(layout="BSND", B=1, S1=3, S2=256, N1=128, topk=128, block_size=1, sparse_mode=0),
    # block-aligned row lists (block size a multiple of 16): 16-row tile loads, padding slots inside
    # the lists (blocks cut by the sequence end or the causal bound, duplicates, -1, blocks past S2)
    "n128_bsnd_bs16_messy": dict(layout="BSND", B=2, S1=5, S2=300, N1=128, topk=20, block_size=16, sparse_mode=3,
                                 index_mode="messy", seqlens_q=[5, 4], seqlens_kv=[300, 37]),
    "n64_tnd_bs32_causal": dict(layout="TND", seqlens_q=[40, 9], seqlens_kv=[200, 70], N1=64, topk=8, block_size=32,
                                sparse_mode=3, index_mode="causal"),
    # every causal block selected (random order, sorted before expansion): rows of up to three
    # contiguous 128-key tiles with a ragged tail; the last sequence's tail tiles reach past the end
    # of the key tensor (601 rows), where the 2-D tile reads zeros
    "n128_tnd_bs16_all_blocks": dict(layout="TND", seqlens_q=[300, 45], seqlens_kv=[300, 301], N1=128, topk=40,
                                     block_size=16, sparse_mode=3, index_mode="causal"),
    # topk below the causal block count for later rows: contiguous and gathered tiles mixed
    "n64_tnd_bs16_mixed_tiles": dict(layout="TND", seqlens_q=[200], seqlens_kv=[200], N1=64, topk=9, block_size=16,
                                     sparse_mode=3, index_mode="causal"),
}


@pytest.mark.parametrize("case", sorted(FUSED))
@pytest.mark.parametrize("det", [False, True])
def test_fused_parity(case, det):
    p = tiny(101, **FUSED[case])
    dp = DevProblem(p)
    out, m, l = prepare_oracle_forward(p, dp)
    got = grads_np(dp.grad_gpu(deterministic=det), p)
    compare_grads(got, oracle_backward(p, out, m, l), what=f"{case}/det={det}/")


def test_fused_fp16():
    p = tiny(103, layout="TND", seqlens_q=[20, 9], seqlens_kv=[200, 150], N1=128, topk=180, block_size=1,
             sparse_mode=3, index_mode="causal")
    for a in (p.q, p.q_rope, p.k, p.k_rope, p.dout):
        a[...] = a.astype(np.float16).astype(np.float32)
    dp = DevProblem(p, dtype=torch.float16)
    out, m, l = prepare_oracle_forward(p, dp)
    compare_grads(grads_np(dp.grad_gpu(), p), oracle_backward(p, out, m, l), what="fused fp16/")


def test_fused_deterministic_bit_identical():
    p = tiny(107, layout="TND", seqlens_q=[60, 90], seqlens_kv=[60, 400], N1=128, topk=30, block_size=16,
             sparse_mode=3, index_mode="causal")
    dp = DevProblem(p)
    prepare_oracle_forward(p, dp)
    a = [r.clone() for r in dp.grad_gpu(deterministic=True)]
    for _ in range(3):
        b = dp.grad_gpu(deterministic=True)
        for x, y in zip(a, b):
            assert torch.equal(x.view(torch.int16), y.view(torch.int16))


def test_fused_matches_generic_path():
    """Same inputs through the fused kernel (value is key) and the CUDA-core
    kernel (value passed as a distinct copy) agree within the bf16 tolerance."""
    p = tiny(109, layout="BSND", B=1, S1=16, S2=500, N1=64, topk=260, block_size=1, sparse_mode=3,
             index_mode="causal")
    dp = DevProblem(p)
    prepare_oracle_forward(p, dp)
    fused = grads_np(dp.grad_gpu(), p)
    dp.v = dp.k.clone()
    generic = grads_np(dp.grad_gpu(), p)
    compare_grads(fused, generic, what="fused-vs-generic/")


FWD = {
    "n128_bsnd_mode0_3tiles": FUSED["n128_bsnd_mode0_bs1_3tiles"],
    "n128_tnd_bs16_causal": FUSED["n128_tnd_bs16_causal"],
    "n128_exact_tile": FUSED["n128_exact_tile"],
    # empty rows (BSND padding positions, all-invalid index lists) and a short ragged tile
    "n128_bsnd_messy_varlen": dict(layout="BSND", B=2, S1=6, S2=150, N1=128, topk=40, block_size=3, sparse_mode=3,
                                   index_mode="messy", seqlens_q=[6, 2], seqlens_kv=[150, 9]),
    # block-aligned row lists (16-row tile loads) with padding slots inside the lists
    "n128_bsnd_bs16_messy": FUSED["n128_bsnd_bs16_messy"],
    "n128_tnd_bs32_causal": dict(layout="TND", seqlens_q=[40, 9], seqlens_kv=[200, 70], N1=128, topk=8, block_size=32,
                                 sparse_mode=3, index_mode="causal"),
    # contiguous 128-key tiles (all causal blocks selected), tails past the end of the key tensor
    "n128_tnd_bs16_all_blocks": FUSED["n128_tnd_bs16_all_blocks"],
    # contiguous and 16-row-tile key loads mixed in one row
    "n128_tnd_bs16_mixed_tiles": dict(FUSED["n64_tnd_bs16_mixed_tiles"], N1=128),
}


@pytest.mark.parametrize("case", sorted(FWD))
def test_fused_fwd_parity(case):
    """Tensor-core forward (N1 = 128, value == key): out, softmaxMax, softmaxSum against the oracle."""
    from parity import assert_close, oracle_forward
    p = tiny(107, **FWD[case])
    dp = DevProblem(p)
    dp.forward_gpu()
    ro, rm, rl = oracle_forward(p)
    go, gm, gl = dp.host_fwd_inputs()
    assert_close("out", go, ro)
    np.testing.assert_allclose(gm, rm, rtol=2e-5, atol=2e-5)
    np.testing.assert_allclose(gl, rl, rtol=2e-5, atol=1e-6)


def test_fused_fwd_running_max_rescale():
    """Key norms that grow with the key index (rows sorted ascending): the running max of
    later tiles exceeds the first tiles' by more than the lazy-rescaling headroom, so the
    accumulated output half and the sum are rescaled during the first output pass."""
    from parity import assert_close, oracle_forward
    from workloads import bf16_round
    p = tiny(111, layout="TND", seqlens_q=[300, 40], seqlens_kv=[300, 500], N1=128, topk=40, block_size=16,
             sparse_mode=3, index_mode="causal")
    f = (1.0 + 8.0 * np.arange(p.T2) / p.T2)[:, None]
    p.k = bf16_round(p.k * f)
    p.k_rope = bf16_round(p.k_rope * f)
    # precondition: for many (row, head) pairs the max over all keys exceeds the first 128-key
    # tile's (keys in ascending order) by more than 8 in log2 units
    from oracle.sfa_oracle import make_spans, selected_rows
    kt = np.concatenate([p.k, p.k_rope], 1)
    moved = 0
    for sp in make_spans(p.layout, p.B, p.S1, p.S2, p.seqlens_q, p.seqlens_kv):
        for pos in range(sp.q_len):
            t = sp.q_start + pos
            rows = sorted(selected_rows(p.indices[t], p.block_size, pos, sp.q_len, sp.kv_len, p.sparse_mode))
            if len(rows) > 128:
                sc = np.concatenate([p.q[t], p.q_rope[t]], 1) @ kt[sp.kv_start + np.array(rows)].T
                moved += int(((sc.max(1) - sc[:, :128].max(1)) * p.scale / np.log(2) > 8).sum())
    assert moved > 1000
    dp = DevProblem(p)
    dp.forward_gpu()
    ro, rm, rl = oracle_forward(p)
    go, gm, gl = dp.host_fwd_inputs()
    assert_close("out", go, ro)
    np.testing.assert_allclose(gm, rm, rtol=2e-5, atol=2e-5)
    np.testing.assert_allclose(gl, rl, rtol=2e-5, atol=1e-6)


def test_fused_fwd_fp16():
    from parity import assert_close, oracle_forward
    p = tiny(109, **FWD["n128_tnd_bs16_causal"])
    for a in (p.q, p.q_rope, p.k, p.k_rope):
        a[...] = a.astype(np.float16).astype(np.float32)
    dp = DevProblem(p, dtype=torch.float16)
    dp.forward_gpu()
    ro, rm, rl = oracle_forward(p)
    go, gm, gl = dp.host_fwd_inputs()
    assert_close("out", go, ro)
    np.testing.assert_allclose(gm, rm, rtol=2e-5, atol=2e-5)
    np.testing.assert_allclose(gl, rl, rtol=2e-5, atol=1e-6)
