"""sfa_grad_noalloc: the backward for callers that cannot allocate device memory.

The entry point takes only inputs and outputs; its scratch is a fixed-size
array inside the library image, shared by all calls on a device.  These tests
call it through the C ABI and compare it with sfa_grad (which takes a caller
workspace) on two different problems in a row, so the second call also proves
that leftovers of the first call in the shared scratch do not leak into its
result.  The size limit is checked on the host, without a GPU.
"""
import ctypes

import pytest
import torch

from sparse_attention_backward_sfa_b200 import _native as N
from workloads import tiny_problem
from parity import DevProblem, compare_grads, grads_np, prepare_oracle_forward

FAKE = ctypes.c_void_p(0x100000)  # never dereferenced: the call fails validation first


def _lib():
    from sparse_attention_backward_sfa_b200 import build
    build.build()
    return N.load()


def _noalloc(lib, dp, det):
    import sparse_attention_backward_sfa_b200 as S
    p = dp.p
    shape = S.sfa_shape(dp.q, dp.k, dp.qr, dp.idx, p.layout, dp.sq)
    outs = (torch.empty_like(dp.q), torch.empty_like(dp.k), torch.empty_like(dp.k), torch.empty_like(dp.qr),
            torch.empty_like(dp.kr))
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    st = lib.sfa_grad_noalloc(P(dp.q), P(dp.k), P(dp.v), P(dp.idx), P(dp.do), P(dp.out), P(dp.smax), P(dp.ssum),
                              P(dp.sq), P(dp.skv), P(dp.qr), P(dp.kr), float(p.scale), p.block_size, p.sparse_mode,
                              0, 0, int(det), ctypes.byref(shape),
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream), *[P(o) for o in outs])
    N.check(st)
    return outs


@pytest.mark.gpu
def test_noalloc_matches_sfa_grad_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = _lib()
    problems = [
        (tiny_problem(801, D=512, Dr=64, layout="TND", seqlens_q=[40, 25], seqlens_kv=[300, 180], N1=128, topk=24,
                      block_size=16, sparse_mode=3, index_mode="causal"), True),
        (tiny_problem(802, D=512, Dr=64, layout="BSND", B=2, S1=9, S2=500, N1=64, topk=200, block_size=1,
                      sparse_mode=0, seqlens_q=[9, 5], seqlens_kv=[500, 260]), False),
    ]
    devs = []
    for p, det in problems:
        dp = DevProblem(p)
        prepare_oracle_forward(p, dp)
        ref = grads_np(dp.grad_gpu(deterministic=det), p)
        got = grads_np(_noalloc(lib, dp, det), p)
        torch.cuda.synchronize()
        compare_grads(got, ref, what=f"noalloc/{p.name}/")
        devs.append((dp, det))
    # deterministic calls are bit-identical run to run, also after another problem has
    # left its contents in the shared scratch
    dp, det = devs[0]
    assert det
    first = [x.clone() for x in _noalloc(lib, dp, True)]
    _noalloc(lib, devs[1][0], devs[1][1])
    again = _noalloc(lib, dp, True)
    torch.cuda.synchronize()
    for name, a, b in zip(("dQuery", "dKey", "dValue", "dQueryRope", "dKeyRope"), first, again):
        assert torch.equal(a, b), f"noalloc deterministic {name} differs between calls"


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = _lib()
    s = N.SfaShape()
    s.layout, s.dtype, s.B, s.S1, s.S2, s.N1, s.N2, s.D, s.Dr, s.topk = 0, 0, 1, 4096, 65536, 128, 1, 512, 64, 2048
    st = lib.sfa_grad_noalloc(*([FAKE] * 10), FAKE, FAKE, 0.04, 1, 0, 0, 0, 1, ctypes.byref(s), None,
                              *([FAKE] * 5))
    assert st == N.SFA_ERR_WORKSPACE
    assert b"limited to" in lib.sfa_last_error_string()
