"""ctypes declarations of the libsfa C ABI (include/sfa.h).

Loading fails loudly: there is no CPU or Python fallback for any entry point.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsfa.so")

SFA_OK = 0
SFA_ERR_NULLPTR = 161001
SFA_ERR_INVALID = 161002
SFA_ERR_WORKSPACE = 161003
SFA_ERR_CUDA = 161004
SFA_ERR_TIMEOUT = 161005
LAYOUT_BSND = 0
LAYOUT_TND = 1
DTYPE_BF16 = 0
DTYPE_FP16 = 1


class SfaShape(ctypes.Structure):
    _fields_ = [("layout", ctypes.c_int32), ("dtype", ctypes.c_int32), ("B", ctypes.c_int64),
                ("S1", ctypes.c_int64), ("S2", ctypes.c_int64), ("T1", ctypes.c_int64), ("T2", ctypes.c_int64),
                ("N1", ctypes.c_int64), ("N2", ctypes.c_int64), ("D", ctypes.c_int64), ("Dr", ctypes.c_int64),
                ("topk", ctypes.c_int64)]


class FaShape(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32), ("B", ctypes.c_int64),
                ("T1", ctypes.c_int64), ("T2", ctypes.c_int64), ("Nq", ctypes.c_int64), ("Nkv", ctypes.c_int64),
                ("D", ctypes.c_int64)]


class LigShape(ctypes.Structure):
    _fields_ = [("layout", ctypes.c_int32), ("dtype", ctypes.c_int32), ("B", ctypes.c_int64),
                ("S1", ctypes.c_int64), ("S2", ctypes.c_int64), ("T1", ctypes.c_int64), ("T2", ctypes.c_int64),
                ("N1", ctypes.c_int64), ("D", ctypes.c_int64), ("Dr", ctypes.c_int64), ("G", ctypes.c_int64),
                ("Di", ctypes.c_int64)]


class SfaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{status}: {msg}")
        self.status = status


_V = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_F = ctypes.c_float
_Dbl = ctypes.c_double
_SZ = ctypes.c_size_t
_PSZ = ctypes.POINTER(ctypes.c_size_t)
_PSH = ctypes.POINTER(SfaShape)
_PFA = ctypes.POINTER(FaShape)
_PLG = ctypes.POINTER(LigShape)

SIGNATURES = {
    "sfa_grad_workspace_size": [_PSH, _I64, _I64, _I32, _PSZ],
    "sfa_grad": [_V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _F, _I64, _I64, _I64, _I64, _I32, _PSH, _V, _SZ,
                 _V, _V, _V, _V, _V, _V],
    "sfa_fwd_workspace_size": [_PSH, _I64, _I64, _PSZ],
    "sfa_fwd": [_V, _V, _V, _V, _V, _V, _V, _V, _F, _I64, _I64, _PSH, _V, _SZ, _V, _V, _V, _V],
    "sfa_compact_indices": [_V, _V, _V, _I64, _I64, _PSH, _V, _V, _V, _V],
    "sfa_key_rows": [_V, _V, _V, _I64, _I64, _PSH, _I32, _I32, _V, _V, _V, _V, _V],
    "sfa_softmax_grad_rowsum": [_V, _V, _PSH, _V, _V],
    "fa_grad_workspace_size": [_PFA, _I64, _I32, _PSZ],
    "fa_grad": [_V, _V, _V, _V, _V, _V, _V, _V, _V, _Dbl, _Dbl, _I64, _I64, _I64, _I64, _I32, _PFA, _V, _SZ, _V,
                _V, _V, _V],
    "fa_fwd_workspace_size": [_PFA, _I64, _PSZ],
    "fa_fwd": [_V, _V, _V, _V, _V, _Dbl, _I64, _PFA, _V, _SZ, _V, _V, _V, _V],
    "sfa_set_kernel_events": [_V, _V],
    "sfa_workspace_status": [_V, _V, ctypes.POINTER(ctypes.c_int32)],
    "sfa_set_wait_limit": [ctypes.c_uint64],
    "sfa_dkv_accum_size": [_PSH, _I32, _PSZ],
    "sfa_grad_rows": [_V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _F, _I64, _I64, _I32, _I64, _I64, _PSH, _V,
                      _SZ, _V, _V, _V, _V, _V],
    "sfa_dout_absmax": [_V, _PSH, _I64, _I64, _V, _V],
    "sfa_dkv_finalize": [_V, _PSH, _I32, _V, _F, _V, _V, _V, _V],
    "sfa_grad_noalloc": [_V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _F, _I64, _I64, _I64, _I64, _I32, _PSH, _V,
                         _V, _V, _V, _V, _V],
    "lig_kl_grad_workspace_size": [_PLG, _I64, _PSZ],
    "lig_kl_grad": [_V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V, _Dbl, _I64, _I64, _I64, _PLG, _V, _SZ, _V,
                    _V, _V, _V, _V],
    "sfa_status_string": [_I32],
    "sfa_last_error_string": [],
    "sfa_version": [],
}
STRING_RESULT = {"sfa_status_string", "sfa_last_error_string", "sfa_version"}

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libsfa.so (once) and declare every exported entry point."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libsfa.so not built at {path}; run __graft_entry__.build() or "
                          f"python -m sparse_attention_backward_sfa_b200.build")
    lib = ctypes.CDLL(path)
    for name, args in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name in STRING_RESULT else ctypes.c_int32
    _lib = lib
    return lib


def check(status: int) -> None:
    if status != SFA_OK:
        lib = load()
        raise SfaError(status, f"{lib.sfa_status_string(status).decode()}: {lib.sfa_last_error_string().decode()}")
