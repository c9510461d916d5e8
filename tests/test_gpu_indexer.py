"""GPU parity of the fused dense lightning-indexer gradient (lig_kl_grad) against the
CPU oracle: several key tiles with a ragged tail, tiles reaching past the end of the
key tensor, causal and full masks, BSND padding rows, rows without a visible key,
N1 = 64 / 128, fp16; then the failure-detection path of the same kernel."""
import numpy as np
import pytest
import torch

from oracle.indexer_kl_oracle import indexer_kl_grad_problem, indexer_softmax_stats
from oracle.sfa_oracle import make_spans, sfa_forward
from workloads import indexer_problem

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_backward_sfa_b200 import build
    build.build()


CASES = {
    # 300-key rows (three tiles, ragged tail); the second sequence's last tiles pass the end of the keys
    "tnd_causal_n128": dict(layout="TND", seqlens_q=[300, 45], seqlens_kv=[300, 301], N1=128, sparse_mode=3),
    # BSND per-batch lengths: padding query rows (zero outputs) and padding key rows (never seen)
    "bsnd_mode0_varlen_n64": dict(layout="BSND", B=2, S1=40, S2=200, seqlens_q=[40, 23], seqlens_kv=[200, 130],
                                  N1=64, sparse_mode=0),
    # S1 > S2 under the causal mask: the first 30 rows see no key
    "tnd_causal_empty_rows": dict(layout="TND", seqlens_q=[50, 20], seqlens_kv=[20, 140], N1=128, sparse_mode=3),
}


def stats(p):
    S2max = max(sp.kv_len for sp in make_spans(p.layout, p.B, p.S1, p.S2, p.seqlens_q, p.seqlens_kv))
    idx = np.tile(np.arange(max(S2max, 1), dtype=np.int32), (p.T1, 1))
    _, m, l = sfa_forward(p.q, p.k, p.k, idx, p.q_rope, p.k_rope, p.scale, 1, p.sparse_mode, p.layout, p.B, p.S1,
                          p.S2, p.seqlens_q, p.seqlens_kv)
    mi, li = indexer_softmax_stats(p.q_index, p.k_index, p.weights, p.layout, p.B, p.S1, p.S2, p.seqlens_q,
                                   p.seqlens_kv, p.sparse_mode)
    # the GPU reads fp32 statistics: the oracle uses the same fp32 values
    return [a.astype(np.float32).astype(np.float64) for a in (m, l, mi, li)]


def device_args(p, dtype=torch.bfloat16):
    dev = "cuda"

    def t(a, shape):
        return torch.tensor(np.asarray(a, np.float32), device=dev).to(dtype).reshape(shape).contiguous()

    if p.layout == "BSND":
        lead_q, lead_k = (p.B, p.S1), (p.B, p.S2)
    else:
        lead_q, lead_k = (p.T1,), (p.T2,)
    q = t(p.q, lead_q + (p.N1, p.D))
    qr = t(p.q_rope, lead_q + (p.N1, p.Dr))
    k = t(p.k, lead_k + (1, p.D))          # one key head
    kr = t(p.k_rope, lead_k + (1, p.Dr))
    qi = t(p.q_index, lead_q + (p.G, p.Di))
    ki = t(p.k_index, lead_k + (1, p.Di))
    w = t(p.weights, lead_q + (p.G,))
    sq = None if p.seqlens_q is None else torch.tensor(p.seqlens_q, dtype=torch.int64, device=dev)
    skv = None if p.seqlens_kv is None else torch.tensor(p.seqlens_kv, dtype=torch.int64, device=dev)
    return q, k, qi, ki, w, qr, kr, sq, skv


def run_gpu(p, st, dtype=torch.bfloat16, workspace=None):
    import sparse_attention_backward_sfa_b200 as S
    q, k, qi, ki, w, qr, kr, sq, skv = device_args(p, dtype)
    m, l, mi, li = (torch.tensor(a, dtype=torch.float32, device="cuda").contiguous() for a in st)
    return S.lig_kl_grad(q, k, qi, ki, w, m, l, mi, li, qr, kr, scale=p.scale, layout=p.layout,
                         sparse_mode=p.sparse_mode, actual_seq_lengths_query=sq, actual_seq_lengths_key=skv,
                         workspace=workspace)


def close(got, ref, what):
    got = np.asarray(got, np.float64).reshape(-1)
    ref = np.asarray(ref, np.float64).reshape(-1)
    assert np.isfinite(got).all(), what
    scale = np.abs(ref).max()
    err = np.abs(got - ref).max()
    assert err <= 2e-2 * scale + 1e-30, f"{what}: max err {err:.3e} vs max |ref| {scale:.3e}"
    if scale > 0:
        cos = float(got @ ref / (np.linalg.norm(got) * np.linalg.norm(ref)))
        assert cos >= 0.9999, f"{what}: cosine {cos:.6f}"


def check(p, dtype=torch.bfloat16):
    st = stats(p)
    dqi, dki, dw, loss = run_gpu(p, st, dtype)
    rq, rk, rw, rl, rows = indexer_kl_grad_problem(p, *st)
    close(dqi.float().cpu().numpy().reshape(p.T1, p.G, p.Di), rq, "dQueryIndex")
    close(dki.float().cpu().numpy().reshape(p.T2, p.Di), rk, "dKeyIndex")
    close(dw.float().cpu().numpy().reshape(p.T1, p.G), rw, "dWeights")
    assert abs(float(loss.item()) - rl) <= 1e-3 * abs(rl) + 1e-6, (float(loss.item()), rl)
    return dqi, dw, rows


@pytest.mark.parametrize("case", sorted(CASES))
def test_indexer_parity(case):
    p = indexer_problem(301, G=64, Di=128, D=512, Dr=64, **CASES[case])
    dqi, dw, rows = check(p)
    # rows without a visible key (padding or masked) are exactly zero
    empty = [sp.q_start + pos for sp in make_spans(p.layout, p.B, p.S1, p.S2, p.seqlens_q, p.seqlens_kv)
             for pos in range(sp.q_len) if (p.sparse_mode == 3 and pos + 1 + sp.kv_len - sp.q_len <= 0)]
    if p.layout == "BSND" and p.seqlens_q is not None:
        empty += [b * p.S1 + i for b in range(p.B) for i in range(int(p.seqlens_q[b]), p.S1)]
    if empty:
        e = torch.tensor(empty, device="cuda")
        assert torch.count_nonzero(dqi.reshape(p.T1, -1)[e]) == 0
        assert torch.count_nonzero(dw.reshape(p.T1, -1)[e]) == 0


def test_indexer_parity_fp16():
    p = indexer_problem(303, layout="TND", seqlens_q=[130, 20], seqlens_kv=[130, 260], N1=128, G=64, Di=128, D=512,
                        Dr=64, sparse_mode=3)
    for name in ("q", "q_rope", "k", "k_rope", "q_index", "k_index", "weights"):
        setattr(p, name, getattr(p, name).astype(np.float16).astype(np.float32))
    check(p, torch.float16)


def test_indexer_wait_timeout_reported_then_recovers():
    """A 1 ns wait limit makes the kernel give up at its first unmet wait: the error word
    reports the site; with the default restored the same context reproduces the result."""
    import sparse_attention_backward_sfa_b200 as S
    p = indexer_problem(305, layout="TND", seqlens_q=[200], seqlens_kv=[200], N1=128, G=64, Di=128, D=512, Dr=64,
                        sparse_mode=3)
    st = stats(p)
    ws = torch.empty(S.lig_kl_grad_workspace_size(S.lig_shape(*device_args(p)[:4], "TND",
                                                              torch.zeros(1, dtype=torch.int64)), 3),
                     dtype=torch.uint8, device="cuda")
    ref = [x.clone() for x in run_gpu(p, st, workspace=ws)]
    assert S.workspace_status(ws) == 0
    try:
        S.set_wait_limit(1)
        run_gpu(p, st, workspace=ws)
        assert S.workspace_status(ws) != 0, "the 1 ns wait limit did not trigger"
    finally:
        S.set_wait_limit(0)
    got = run_gpu(p, st, workspace=ws)
    assert S.workspace_status(ws) == 0
    # dKeyIndex uses fp32 atomics (order may differ); the other outputs are per-row and exact
    assert torch.equal(got[0], ref[0]) and torch.equal(got[2], ref[2]) and torch.equal(got[3], ref[3])
    torch.testing.assert_close(got[1].float(), ref[1].float(), rtol=1e-2, atol=1e-3)
