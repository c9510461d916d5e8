"""Failure detection without a GPU fault: with the device-side wait limit set to 1 ns,
each fused kernel gives up at its first wait that is not already satisfied, records the
wait site in its workspace's error word, drains what it issued, frees its tensor memory
and exits; sfa_workspace_status reports it (SFA_ERR_TIMEOUT).  With the default limit
restored, the same CUDA context then computes the same results as before."""
import numpy as np
import pytest
import torch

from workloads import tiny_problem, make_fa_problem
from parity import DevFA, DevProblem, prepare_oracle_forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_backward_sfa_b200 import build
    build.build()


@pytest.fixture(autouse=True)
def _restore_limit():
    yield
    import sparse_attention_backward_sfa_b200 as S
    S.set_wait_limit(0)


def _ws(nbytes):
    return torch.empty(nbytes, dtype=torch.uint8, device="cuda")


def test_sfa_backward_wait_timeout_reported_then_recovers():
    import sparse_attention_backward_sfa_b200 as S
    p = tiny_problem(401, D=512, Dr=64, layout="TND", seqlens_q=[70, 3, 150], seqlens_kv=[70, 260, 150], N1=128,
                     topk=12, block_size=16, sparse_mode=3, index_mode="causal")
    dp = DevProblem(p)
    prepare_oracle_forward(p, dp)
    shape = S.sfa_shape(dp.q, dp.k, dp.qr, dp.idx, p.layout, dp.sq)
    ws = _ws(S.sfa_grad_workspace_size(shape, p.block_size, p.sparse_mode, True))
    ref = [t.clone() for t in dp.grad_gpu(deterministic=True, workspace=ws)]
    assert S.workspace_status(ws) == 0
    S.set_wait_limit(1)
    dp.grad_gpu(deterministic=True, workspace=ws)
    site = S.workspace_status(ws)
    assert site != 0, "the 1 ns wait limit did not trigger"
    S.set_wait_limit(0)
    got = dp.grad_gpu(deterministic=True, workspace=ws)
    assert S.workspace_status(ws) == 0
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


def test_sfa_forward_wait_timeout_reported_then_recovers():
    import ctypes
    import sparse_attention_backward_sfa_b200 as S
    from sparse_attention_backward_sfa_b200 import _native as N
    p = tiny_problem(403, D=512, Dr=64, layout="BSND", B=1, S1=5, S2=700, N1=128, topk=300, block_size=1,
                     sparse_mode=0)
    dp = DevProblem(p)
    shape = S.sfa_shape(dp.q, dp.k, dp.qr, dp.idx, p.layout, dp.sq)
    n = ctypes.c_size_t()
    N.check(N.load().sfa_fwd_workspace_size(ctypes.byref(shape), p.block_size, p.sparse_mode, ctypes.byref(n)))
    ws = _ws(n.value)
    ref = [t.clone() for t in S.sfa_fwd(dp.q, dp.k, dp.v, dp.idx, dp.qr, dp.kr, workspace=ws, **dp.kw())]
    assert S.workspace_status(ws) == 0
    S.set_wait_limit(1)
    S.sfa_fwd(dp.q, dp.k, dp.v, dp.idx, dp.qr, dp.kr, workspace=ws, **dp.kw())
    assert S.workspace_status(ws) != 0, "the 1 ns wait limit did not trigger"
    S.set_wait_limit(0)
    got = S.sfa_fwd(dp.q, dp.k, dp.v, dp.idx, dp.qr, dp.kr, workspace=ws, **dp.kw())
    assert S.workspace_status(ws) == 0
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


def test_fa_backward_wait_timeout_reported_then_recovers():
    import ctypes
    import sparse_attention_backward_sfa_b200 as S
    from sparse_attention_backward_sfa_b200 import _native as N
    fp = make_fa_problem(seed=405, lens=(130, 70), N=4, Nkv=2, D=128)
    d = DevFA(fp)
    d.forward_gpu()
    shape = S.ops._fa_shape(d.q, d.k, fp.cu_seqlens_q, fp.cu_seqlens_kv)
    n = ctypes.c_size_t()
    N.check(N.load().fa_grad_workspace_size(ctypes.byref(shape), 3, 1, ctypes.byref(n)))
    ws = _ws(n.value)
    ref = [t.clone() for t in d.grad_gpu(deterministic=True, workspace=ws)]
    assert S.workspace_status(ws) == 0
    S.set_wait_limit(1)
    d.grad_gpu(deterministic=True, workspace=ws)
    assert S.workspace_status(ws) != 0, "the 1 ns wait limit did not trigger"
    S.set_wait_limit(0)
    got = d.grad_gpu(deterministic=True, workspace=ws)
    assert S.workspace_status(ws) == 0
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
