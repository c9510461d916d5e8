"""Pins of the dense lightning-indexer gradient oracle (DenseLightningIndexerGradKLLoss,
功能说明 formulas 1-4) against things other than itself:

* finite differences of the loss (KL of the head-averaged main-attention distribution
  against softmax(I), with softmax(I) recomputed from I at every evaluation) give
  dq~I, dK~I and dW;
* torch fp64 autograd of the same loss written with library routines
  (``torch.softmax``, ``torch.log_softmax``, ``torch.nn.functional.kl_div``) gives the loss
  value and the three gradients;
* when the indexer's distribution equals the target one the divergence and every
  gradient vanish.
"""
import numpy as np
import pytest
import torch

from oracle.indexer_kl_oracle import indexer_kl_grad_problem, indexer_softmax_stats, visible_keys
from oracle.sfa_oracle import make_spans, sfa_forward
from workloads import indexer_problem

CASES = {
    "tnd_causal": dict(layout="TND", seqlens_q=[5, 3], seqlens_kv=[7, 3], N1=2, G=3, Di=4, D=6, Dr=2, sparse_mode=3),
    "bsnd_mode0_varlen": dict(layout="BSND", B=2, S1=3, S2=5, seqlens_q=[3, 2], seqlens_kv=[5, 4], N1=3, G=2, Di=3,
                              D=4, Dr=2, sparse_mode=0),
}


def main_stats(p):
    """softmaxMax / softmaxSum of the main attention over every visible key (the
    sparse-attention forward oracle with an index table listing all key rows)."""
    S2max = max(sp.kv_len for sp in make_spans(p.layout, p.B, p.S1, p.S2, p.seqlens_q, p.seqlens_kv))
    idx = np.tile(np.arange(S2max, dtype=np.int32), (p.T1, 1))
    _, m, l = sfa_forward(p.q, p.k, p.k, idx, p.q_rope, p.k_rope, p.scale, 1, p.sparse_mode, p.layout, p.B, p.S1,
                          p.S2, p.seqlens_q, p.seqlens_kv)
    return m, l


def run(p, m, l, qi=None, ki=None, w=None):
    """Oracle loss and gradients with the indexer statistics recomputed from I."""
    import dataclasses
    p2 = dataclasses.replace(p, q_index=p.q_index if qi is None else qi, k_index=p.k_index if ki is None else ki,
                             weights=p.weights if w is None else w)
    mi, li = indexer_softmax_stats(p2.q_index, p2.k_index, p2.weights, p2.layout, p2.B, p2.S1, p2.S2, p2.seqlens_q,
                                   p2.seqlens_kv, p2.sparse_mode)
    return indexer_kl_grad_problem(p2, m, l, mi, li)


@pytest.mark.parametrize("case", sorted(CASES))
def test_finite_differences(case):
    p = indexer_problem(11, round_bf16=False, **CASES[case])
    m, l = main_stats(p)
    dqi, dki, dw, _, _ = run(p, m, l)
    eps = 1e-6
    for name, base, grad in (("q_index", p.q_index, dqi), ("k_index", p.k_index, dki), ("weights", p.weights, dw)):
        fd = np.zeros_like(base)
        for i in np.ndindex(base.shape):
            hi, lo = base.copy(), base.copy()
            hi[i] += eps
            lo[i] -= eps
            kw_hi = {name.replace("q_index", "qi").replace("k_index", "ki").replace("weights", "w"): hi}
            kw_lo = {name.replace("q_index", "qi").replace("k_index", "ki").replace("weights", "w"): lo}
            fd[i] = (run(p, m, l, **kw_hi)[3] - run(p, m, l, **kw_lo)[3]) / (2 * eps)
        np.testing.assert_allclose(grad, fd, rtol=1e-5, atol=1e-7, err_msg=f"{case}: d{name}")


def torch_reference(p):
    """Loss and gradients from torch fp64 autograd: per-head softmax of the masked
    main scores averaged over heads as the target, log_softmax of the indexer
    scores, kl_div(reduction='sum')."""
    qi = torch.tensor(p.q_index, dtype=torch.float64, requires_grad=True)
    ki = torch.tensor(p.k_index, dtype=torch.float64, requires_grad=True)
    w = torch.tensor(p.weights, dtype=torch.float64, requires_grad=True)
    qt = torch.cat([torch.tensor(p.q, dtype=torch.float64), torch.tensor(p.q_rope, dtype=torch.float64)], dim=2)
    kt = torch.cat([torch.tensor(p.k, dtype=torch.float64), torch.tensor(p.k_rope, dtype=torch.float64)], dim=1)
    loss = torch.zeros((), dtype=torch.float64)
    for sp in make_spans(p.layout, p.B, p.S1, p.S2, p.seqlens_q, p.seqlens_kv):
        for pos in range(sp.q_len):
            t = sp.q_start + pos
            n = visible_keys(pos, sp.q_len, sp.kv_len, p.sparse_mode)
            if n == 0:
                continue
            rows = slice(sp.kv_start, sp.kv_start + n)
            target = torch.softmax(p.scale * qt[t] @ kt[rows].T, dim=1).mean(dim=0)
            scores = (w[t][:, None] * torch.relu(qi[t] @ ki[rows].T)).sum(dim=0)
            loss = loss + torch.nn.functional.kl_div(torch.log_softmax(scores, dim=0), target, reduction="sum")
    loss.backward()
    return float(loss.detach()), qi.grad.numpy(), ki.grad.numpy(), w.grad.numpy()


@pytest.mark.parametrize("case", sorted(CASES))
def test_torch_autograd_special_case(case):
    p = indexer_problem(12, round_bf16=False, **CASES[case])
    m, l = main_stats(p)
    dqi, dki, dw, loss, loss_t = run(p, m, l)
    tl, tqi, tki, tw = torch_reference(p)
    assert loss > 0
    np.testing.assert_allclose(loss, tl, rtol=1e-10)
    np.testing.assert_allclose(loss_t.sum(), tl, rtol=1e-10)
    np.testing.assert_allclose(dqi, tqi, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dki, tki, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dw, tw, rtol=1e-9, atol=1e-12)


def test_zero_divergence_when_distributions_match():
    """One main head and one indexer head whose score is the main scaled score plus
    a constant (q~I = [Q~, c], K~I = [scale K~, c], W = 1, every dot product > 0):
    softmax(I) equals the target, so the loss and all gradients are zero."""
    p = indexer_problem(13, layout="TND", seqlens_q=[4, 6], seqlens_kv=[4, 9], N1=1, G=1, Di=1, D=5, Dr=3,
                        sparse_mode=3, round_bf16=False)
    c = 30.0
    qt = np.concatenate([p.q[:, 0, :], p.q_rope[:, 0, :]], axis=1)                 # [T1, 8]
    kt = np.concatenate([p.k, p.k_rope], axis=1) * p.scale                          # [T2, 8]
    p.q_index = np.concatenate([qt, np.full((p.T1, 1), c)], axis=1)[:, None, :]    # [T1, 1, 9]
    p.k_index = np.concatenate([kt, np.full((p.T2, 1), c)], axis=1)                # [T2, 9]
    p.weights = np.ones((p.T1, 1))
    p.Di = 9
    assert (p.q_index[:, 0, :] @ p.k_index.T).min() > 0
    m, l = main_stats(p)
    dqi, dki, dw, loss, _ = run(p, m, l)
    assert abs(loss) < 1e-12
    for g in (dqi, dki, dw):
        assert np.abs(g).max() < 1e-12
