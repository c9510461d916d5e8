"""C ABI checks that need no GPU: the library loads, exports every entry point
declared in include/sfa.h, and rejects bad arguments on the host (before any
launch) with the documented status codes."""
import ctypes
import os
import re

import pytest

from sparse_attention_backward_sfa_b200 import _native as N
from sparse_attention_backward_sfa_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return N.load()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "sfa.h")).read()
    return sorted(set(re.findall(r"^(?:sfa_status|const char \*)\s*(\w+)\s*\(", src, re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("sfa_grad", "sfa_grad_workspace_size", "sfa_fwd", "fa_grad", "fa_fwd", "sfa_compact_indices",
              "sfa_softmax_grad_rowsum", "sfa_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(lib, n), n
        assert n in N.SIGNATURES, f"binding lacks {n}"


def test_status_strings(lib):
    assert lib.sfa_status_string(N.SFA_OK) == b"SFA_OK"
    assert lib.sfa_status_string(N.SFA_ERR_INVALID) == b"SFA_ERR_INVALID"
    assert lib.sfa_version().startswith(b"0.")


def _shape(**kw):
    s = N.SfaShape()
    d = dict(layout=0, dtype=0, B=1, S1=128, S2=2048, T1=0, T2=0, N1=128, N2=1, D=512, Dr=64, topk=1024)
    d.update(kw)
    for k, v in d.items():
        setattr(s, k, v)
    return s


@pytest.mark.parametrize("kw,bs,mode,code", [
    ({}, 1, 0, N.SFA_OK),
    (dict(N2=2), 1, 0, N.SFA_ERR_INVALID),
    (dict(D=256), 1, 0, N.SFA_ERR_INVALID),
    (dict(Dr=32), 1, 0, N.SFA_ERR_INVALID),
    (dict(N1=5), 1, 0, N.SFA_ERR_INVALID),
    (dict(N1=48), 1, 0, N.SFA_OK),
    (dict(B=0), 1, 0, N.SFA_ERR_INVALID),
    (dict(B=257), 1, 0, N.SFA_ERR_INVALID),
    (dict(S1=128 * 1024 + 1), 1, 0, N.SFA_ERR_INVALID),
    (dict(layout=2), 1, 0, N.SFA_ERR_INVALID),
    (dict(dtype=3), 1, 0, N.SFA_ERR_INVALID),
    (dict(topk=0), 1, 0, N.SFA_ERR_INVALID),
    ({}, 0, 0, N.SFA_ERR_INVALID),
    ({}, 1, 1, N.SFA_ERR_INVALID),
    ({}, 16, 3, N.SFA_OK),
    (dict(layout=1, T1=100, T2=100, B=2), 1, 3, N.SFA_OK),
    (dict(layout=1, T1=0, T2=100, B=2), 1, 3, N.SFA_ERR_INVALID),
])
def test_workspace_size_validation(lib, kw, bs, mode, code):
    n = ctypes.c_size_t(0)
    sh = _shape(**kw)
    assert lib.sfa_grad_workspace_size(ctypes.byref(sh), bs, mode, 0, ctypes.byref(n)) == code
    if code == N.SFA_OK:
        assert n.value > 0
    else:
        assert lib.sfa_last_error_string()


def test_deterministic_workspace_is_larger(lib):
    sh = _shape()
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    lib.sfa_grad_workspace_size(ctypes.byref(sh), 1, 0, 0, ctypes.byref(a))
    lib.sfa_grad_workspace_size(ctypes.byref(sh), 1, 0, 1, ctypes.byref(b))
    assert b.value > a.value


FAKE = ctypes.c_void_p(0x100000)  # never dereferenced: every case fails validation first


def _grad_call(lib, sh, ws_bytes, **over):
    args = dict(q=FAKE, k=FAKE, v=FAKE, idx=FAKE, do=FAKE, o=FAKE, mx=FAKE, sm=FAKE, sq=None, skv=None, qr=FAKE,
                kr=FAKE, ws=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, dqr=FAKE, dkr=FAKE)
    args.update(over)
    a = args
    return lib.sfa_grad(a["q"], a["k"], a["v"], a["idx"], a["do"], a["o"], a["mx"], a["sm"], a["sq"], a["skv"],
                        a["qr"], a["kr"], 0.04, 1, 0, 0, 0, 0, ctypes.byref(sh), a["ws"], ws_bytes, None, a["dq"],
                        a["dk"], a["dv"], a["dqr"], a["dkr"])


def test_grad_host_errors(lib):
    sh = _shape()
    assert _grad_call(lib, sh, 1 << 40, q=None) == N.SFA_ERR_NULLPTR
    assert _grad_call(lib, sh, 1 << 40, dkr=None) == N.SFA_ERR_NULLPTR
    assert _grad_call(lib, sh, 16) == N.SFA_ERR_WORKSPACE
    assert b"workspace" in lib.sfa_last_error_string()
    assert _grad_call(lib, sh, 1 << 40, ws=ctypes.c_void_p(0x100010)) == N.SFA_ERR_INVALID
    tnd = _shape(layout=1, T1=64, T2=64, B=1)
    assert _grad_call(lib, tnd, 1 << 40) == N.SFA_ERR_NULLPTR  # TND without seqlens
    assert _grad_call(lib, _shape(D=128), 1 << 40) == N.SFA_ERR_INVALID


def test_fa_host_errors(lib):
    s = N.FaShape()
    s.dtype, s.B, s.T1, s.T2, s.Nq, s.Nkv, s.D = 0, 1, 256, 256, 16, 4, 128
    n = ctypes.c_size_t()
    assert lib.fa_grad_workspace_size(ctypes.byref(s), 3, 0, ctypes.byref(n)) == N.SFA_OK
    s.Nkv = 3
    assert lib.fa_grad_workspace_size(ctypes.byref(s), 3, 0, ctypes.byref(n)) == N.SFA_ERR_INVALID
    s.Nkv = 4
    s.D = 260
    assert lib.fa_grad_workspace_size(ctypes.byref(s), 3, 0, ctypes.byref(n)) == N.SFA_ERR_INVALID
    s.D = 128
    cu = (ctypes.c_int64 * 1)(255)  # last entry must equal T
    ok = (ctypes.c_int64 * 1)(256)
    st = lib.fa_grad(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, cu, ok, 0.08, 1.0, 0, 0, 16, 3, 0, ctypes.byref(s),
                     FAKE, 1 << 40, None, FAKE, FAKE, FAKE)
    assert st == N.SFA_ERR_INVALID
    st = lib.fa_grad(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ok, ok, 0.08, 0.9, 0, 0, 16, 3, 0, ctypes.byref(s),
                     FAKE, 1 << 40, None, FAKE, FAKE, FAKE)
    assert st == N.SFA_ERR_INVALID  # keep_prob != 1
    st = lib.fa_grad(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ok, ok, 0.08, 1.0, 0, 0, 8, 3, 0, ctypes.byref(s),
                     FAKE, 1 << 40, None, FAKE, FAKE, FAKE)
    assert st == N.SFA_ERR_INVALID  # head_num != Nq


def _lig_shape(**kw):
    s = N.LigShape()
    d = dict(layout=0, dtype=0, B=1, S1=64, S2=256, T1=0, T2=0, N1=128, D=512, Dr=64, G=64, Di=128)
    d.update(kw)
    for k, v in d.items():
        setattr(s, k, v)
    return s


@pytest.mark.parametrize("kw,mode,code", [
    ({}, 3, N.SFA_OK),
    ({}, 0, N.SFA_OK),
    (dict(N1=64), 3, N.SFA_OK),
    (dict(layout=1, T1=300, T2=300, B=2), 3, N.SFA_OK),
    ({}, 1, N.SFA_ERR_INVALID),
    (dict(N1=32), 3, N.SFA_ERR_INVALID),
    (dict(G=32), 3, N.SFA_ERR_INVALID),
    (dict(Di=64), 3, N.SFA_ERR_INVALID),
    (dict(D=256), 3, N.SFA_ERR_INVALID),
    (dict(B=0), 3, N.SFA_ERR_INVALID),
    (dict(layout=2), 3, N.SFA_ERR_INVALID),
    (dict(dtype=2), 3, N.SFA_ERR_INVALID),
    (dict(layout=1, T1=0, T2=10, B=1), 3, N.SFA_ERR_INVALID),
])
def test_lig_workspace_size_validation(lib, kw, mode, code):
    n = ctypes.c_size_t(0)
    sh = _lig_shape(**kw)
    assert lib.lig_kl_grad_workspace_size(ctypes.byref(sh), mode, ctypes.byref(n)) == code
    if code == N.SFA_OK:
        T2 = sh.T2 if sh.layout == 1 else sh.B * sh.S2
        assert n.value >= T2 * 128 * 4  # holds the fp32 dKeyIndex accumulator


def test_lig_rejects_null_pointers_before_launch(lib):
    sh = _lig_shape()
    n = ctypes.c_size_t(0)
    assert lib.lig_kl_grad_workspace_size(ctypes.byref(sh), 3, ctypes.byref(n)) == N.SFA_OK
    args = [None] * 13 + [0.05, 3, 0, 0, ctypes.byref(sh), None, n.value, None] + [None] * 4
    assert lib.lig_kl_grad(*args) == N.SFA_ERR_NULLPTR
    assert lib.lig_kl_grad_workspace_size(None, 3, ctypes.byref(n)) == N.SFA_ERR_NULLPTR


def test_lig_shape_reads_rope_width_from_the_tensor(lib):
    """The binding takes Dr from queryRope, so a wrong rope width reaches the library's check."""
    import torch
    from sparse_attention_backward_sfa_b200 import ops
    q = torch.empty(10, 128, 512, dtype=torch.bfloat16)
    k = torch.empty(10, 1, 512, dtype=torch.bfloat16)
    qi = torch.empty(10, 64, 128, dtype=torch.bfloat16)
    ki = torch.empty(10, 1, 128, dtype=torch.bfloat16)
    sq = torch.tensor([10], dtype=torch.int64)
    good = ops.lig_shape(q, k, qi, ki, "TND", sq, torch.empty(10, 128, 64, dtype=torch.bfloat16))
    bad = ops.lig_shape(q, k, qi, ki, "TND", sq, torch.empty(10, 128, 32, dtype=torch.bfloat16))
    n = ctypes.c_size_t(0)
    assert lib.lig_kl_grad_workspace_size(ctypes.byref(good), 3, ctypes.byref(n)) == N.SFA_OK
    assert lib.lig_kl_grad_workspace_size(ctypes.byref(bad), 3, ctypes.byref(n)) == N.SFA_ERR_INVALID
