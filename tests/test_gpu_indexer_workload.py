"""The indexer-gradient benchmark workload at full size (TND {2048, 4096, 4096, 6144},
N1 = 128, G = 64, Di = 128, causal), in the launch configuration bench.py times,
checked against the oracle on a seeded sample of query rows:
 (i)  dQueryIndex / dWeights rows of the sampled tokens from the full run;
 (ii) a second full run whose weights are zero outside the sample (those rows then
      contribute exactly nothing to dKeyIndex) against the oracle's dKeyIndex summed
      over the sampled rows.
The statistics are the benchmark's (sfa_fwd over every causal block for the main
attention, the indexer's max / sum over its visible keys)."""
import numpy as np
import pytest
import torch

from oracle import indexer_kl_oracle as O
from workloads import RowView

pytestmark = pytest.mark.gpu

N_SAMPLE = 128


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_backward_sfa_b200 import build
    build.build()


def close(got, ref, what):
    got = np.asarray(got, np.float64).reshape(-1)
    ref = np.asarray(ref, np.float64).reshape(-1)
    assert np.isfinite(got).all(), what
    scale = np.abs(ref).max()
    err = np.abs(got - ref).max()
    assert err <= 2e-2 * scale, f"{what}: max err {err:.3e} vs max |ref| {scale:.3e}"
    cos = float(got @ ref / (np.linalg.norm(got) * np.linalg.norm(ref)))
    assert cos >= 0.9999, f"{what}: cosine {cos:.6f}"


def test_indexer_workload_sampled():
    import bench
    import sparse_attention_backward_sfa_b200 as S
    dev = torch.device("cuda", 0)
    p, lens, smax, ssum, mi, li = bench.indexer_inputs(dev)
    kw = dict(scale=p.scale, layout="TND", sparse_mode=3, actual_seq_lengths_query=p.seqlens_q,
              actual_seq_lengths_key=p.seqlens_kv)
    dqi, _, dw, loss = S.lig_kl_grad(p.q, p.k, p.q_index, p.k_index, p.weights, smax, ssum, mi, li, p.q_rope,
                                     p.k_rope, **kw)
    assert torch.isfinite(loss).all() and float(loss.item()) > 0
    rng = np.random.default_rng(p.meta["seed"] + 1)
    toks = np.sort(rng.choice(p.T1, size=N_SAMPLE, replace=False))
    sel = torch.tensor(toks, device=dev)
    mask = torch.zeros(p.T1, dtype=p.weights.dtype, device=dev)
    mask[sel] = 1
    w2 = (p.weights * mask[:, None]).contiguous()
    _, dki2, _, _ = S.lig_kl_grad(p.q, p.k, p.q_index, p.k_index, w2, smax, ssum, mi, li, p.q_rope, p.k_rope, **kw)

    T1, T2 = p.T1, p.T2
    views = [RowView(x, toks, T1) for x in (p.q, p.q_rope, p.q_index, p.weights, smax, ssum, mi.reshape(T1, 1),
                                            li.reshape(T1, 1))]
    qv, qrv, qiv, wv, mv, lv, miv, liv = views
    k = p.k.reshape(T2, p.D).float().cpu().numpy()
    kr = p.k_rope.reshape(T2, p.Dr).float().cpu().numpy()
    ki = p.k_index.reshape(T2, p.Di).float().cpu().numpy()
    sq = p.seqlens_q.cpu().numpy()
    rq, rk, rw, _, _ = O.indexer_kl_grad(qv, k, qiv, ki, wv, mv, lv, miv, liv, qrv, kr, p.scale, "TND", p.B, 0, 0,
                                         sq, sq, 3, tokens=toks)
    close(dqi.reshape(T1, p.G, p.Di)[sel].float().cpu().numpy(), rq[toks], "dQueryIndex (sampled rows)")
    close(dw.reshape(T1, p.G)[sel].float().cpu().numpy(), rw[toks], "dWeights (sampled rows)")
    close(dki2.reshape(T2, p.Di).float().cpu().numpy(), rk, "dKeyIndex (sampled rows' contributions)")
