"""Full-size workloads 3, 4, 5 on the GPU, checked against the oracle on a seeded
sample of 256 query rows:
 (i)  dQuery / dQueryRope rows of the sampled tokens from the full run,
 (ii) a second full-size run whose dO is zero outside the sample (those rows then
      contribute exactly nothing) against the oracle's dKey / dValue / dKeyRope
      summed over the sampled rows,
 (iii) for the deterministic workload, two full runs bit for bit.
O and the softmax statistics come from the library's forward; the oracle
checks the forward on the same sampled rows."""
import numpy as np
import pytest
import torch

from oracle import sfa_oracle as O
from workloads import RowView, make_device_problem
from parity import assert_close

pytestmark = pytest.mark.gpu

N_SAMPLE = 256


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_backward_sfa_b200 import build
    build.build()


def _kw(p):
    return dict(scale=p.scale, sparse_block_size=p.block_size, layout=p.layout, sparse_mode=p.sparse_mode,
                actual_seq_lengths_q=p.seqlens_q, actual_seq_lengths_kv=p.seqlens_kv)


def _host(x):
    return None if x is None else x.cpu().numpy()


@pytest.mark.parametrize("cfg", [3, 4, 5])
def test_workload_sampled(cfg):
    import sparse_attention_backward_sfa_b200 as S
    p = make_device_problem(cfg)
    out, smax, ssum = S.sfa_fwd(p.q, p.k, p.k, p.indices, p.q_rope, p.k_rope, **_kw(p))
    res = S.sfa_grad(p.q, p.k, p.k, p.indices, p.dout, out, smax, ssum, p.q_rope, p.k_rope,
                     deterministic=p.deterministic, **_kw(p))
    dq_full = res[0].reshape(p.T1, p.N1, p.D)
    dqr_full = res[3].reshape(p.T1, p.N1, p.Dr)
    rng = np.random.default_rng(p.meta["seed"] + 1)
    toks = np.sort(rng.choice(p.T1, size=N_SAMPLE, replace=False))
    sel = torch.tensor(toks, device=p.q.device)

    # (ii) rerun with dO zero outside the sample
    mask = torch.zeros(p.T1, dtype=torch.bool, device=p.q.device)
    mask[sel] = True
    do_masked = (p.dout.reshape(p.T1, -1) * mask[:, None]).reshape(p.dout.shape)
    res2 = S.sfa_grad(p.q, p.k, p.k, p.indices, do_masked, out, smax, ssum, p.q_rope, p.k_rope,
                      deterministic=p.deterministic, **_kw(p))

    # oracle on the sampled rows (fp64)
    T1 = p.T1
    qv = RowView(p.q, toks, T1)
    qrv = RowView(p.q_rope, toks, T1)
    dov = RowView(p.dout, toks, T1)
    ov = RowView(out, toks, T1)
    mv = RowView(smax, toks, T1)
    lv = RowView(ssum, toks, T1)
    iv = RowView(p.indices, toks, T1)
    k = p.k.reshape(p.T2, p.D).float().cpu().numpy()
    kr = p.k_rope.reshape(p.T2, p.Dr).float().cpu().numpy()
    sq, skv = _host(p.seqlens_q), _host(p.seqlens_kv)
    ro, rm, rl = O.sfa_forward(qv, k, k, iv, qrv, kr, p.scale, p.block_size, p.sparse_mode, p.layout, p.B, p.S1,
                               p.S2, sq, skv, tokens=toks)
    assert_close(f"cfg{cfg} out", np.stack([ov[t] for t in toks]), ro)
    np.testing.assert_allclose(np.stack([mv[t] for t in toks]), rm, rtol=1e-4, atol=1e-4)
    np.testing.assert_allclose(np.stack([lv[t] for t in toks]), rl, rtol=1e-4, atol=1e-5)
    rq, rk, rvv, rqr, rkr = O.sfa_backward(qv, k, k, iv, dov, ov, mv, lv, qrv, kr, p.scale, p.block_size,
                                           p.sparse_mode, p.layout, p.B, p.S1, p.S2, sq, skv, tokens=toks)
    assert_close(f"cfg{cfg} dQuery (full run, sampled rows)", dq_full[sel].float().cpu().numpy(), rq)
    assert_close(f"cfg{cfg} dQueryRope (full run, sampled rows)", dqr_full[sel].float().cpu().numpy(), rqr)
    assert_close(f"cfg{cfg} dKey (sub-problem)", res2[1].reshape(p.T2, p.D).float().cpu().numpy(), rk)
    assert_close(f"cfg{cfg} dValue (sub-problem)", res2[2].reshape(p.T2, p.D).float().cpu().numpy(), rvv)
    assert_close(f"cfg{cfg} dKeyRope (sub-problem)", res2[4].reshape(p.T2, p.Dr).float().cpu().numpy(), rkr)
    assert_close(f"cfg{cfg} dQuery (sub-problem rows)",
                 res2[0].reshape(p.T1, p.N1, p.D)[sel].float().cpu().numpy(), rq)

    if p.deterministic:
        res3 = S.sfa_grad(p.q, p.k, p.k, p.indices, p.dout, out, smax, ssum, p.q_rope, p.k_rope,
                          deterministic=True, **_kw(p))
        for a, b in zip(res, res3):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))
