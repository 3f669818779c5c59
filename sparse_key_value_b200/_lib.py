"""ctypes binding of libpkm.so (argument marshalling only).

Every step of the lookup runs in the library's CUDA kernels; this module
only turns torch tensors into pointers and sizes and raises on a non-OK
status.  It fails loudly if the library is missing: there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libpkm.so")

PKM_OK = 0
STATUS = {0: "PKM_OK", 1: "PKM_ERR_INVALID_ARG", 2: "PKM_ERR_UNSUPPORTED", 3: "PKM_ERR_CUDA",
          4: "PKM_ERR_DEVICE", 5: "PKM_ERR_TIMEOUT", 6: "PKM_ERR_WORKSPACE"}
PKM_F32, PKM_BF16 = 0, 1

P = ctypes.c_void_p
I32, I64, SZ = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t


class PKMError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)}")


class FwdArgs(ctypes.Structure):
    _fields_ = [("T", I64), ("H", I32), ("d_half", I32), ("n_sub", I32), ("k", I32),
                ("d_v", I32), ("dtype", ctypes.c_int), ("query", P), ("subkeys", P),
                ("values", P), ("x", P), ("W1", P), ("W2", P), ("d_model", I32), ("out", P),
                ("idx", P), ("weights", P), ("workspace", P), ("workspace_bytes", SZ),
                ("phase_events", P), ("y_out", P)]


FWD_N_EVENTS = 7


class BwdArgs(ctypes.Structure):
    _fields_ = [("T", I64), ("H", I32), ("d_half", I32), ("n_sub", I32), ("k", I32),
                ("d_v", I32), ("dtype", ctypes.c_int), ("query", P), ("subkeys", P),
                ("values", P), ("idx", P), ("weights", P), ("dy", P), ("dquery", P),
                ("dsubkeys", P), ("uniq_rows", P), ("grad_rows", P), ("n_uniq", P),
                ("uniq_cap", I64), ("dvalues_dense", P), ("dscores", P), ("workspace", P),
                ("workspace_bytes", SZ)]


class MemplusBwdArgs(ctypes.Structure):
    _fields_ = [("T", I64), ("d_model", I32), ("d_v", I32), ("x", P), ("W1", P), ("W2", P),
                ("y", P), ("dout", P), ("dy", P), ("dx", P), ("dW1", P), ("dW2", P),
                ("workspace", P), ("workspace_bytes", SZ)]


class QprojArgs(ctypes.Structure):
    _fields_ = [("T", I64), ("d_model", I32), ("d_q", I32), ("x", P), ("Wq", P), ("q", P),
                ("dq", P), ("dWq", P), ("dx", P), ("workspace", P), ("workspace_bytes", SZ)]


class SparseOptArgs(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("lr", ctypes.c_float), ("beta1", ctypes.c_float),
                ("beta2", ctypes.c_float), ("eps", ctypes.c_float), ("step", I64),
                ("n_rows", I64), ("d", I32), ("dtype", ctypes.c_int), ("table", P), ("rows", P),
                ("grads", P), ("count", P), ("cap", I64), ("m", P), ("v", P)]


class EngramArgs(ctypes.Structure):
    _fields_ = [("n_seq", I64), ("L", I32), ("n_orders", I32), ("K", I32), ("orders", P),
                ("seeds", P), ("rows_per_head", P), ("d", I32), ("dtype", ctypes.c_int),
                ("tokens", P), ("table", P), ("h", P), ("v", P), ("alpha", P), ("rows", P),
                ("e", P)]


EXPORTS = ("pkm_forward_workspace_size", "pkm_forward", "pkm_backward_workspace_size",
           "pkm_backward", "embbag_forward", "embbag_backward_workspace_size",
           "embbag_backward", "pkm_get_device_error", "pkm_status_string", "pkm_version",
           "pkm_launch_count", "pkm_forward_noalloc", "pkm_memplus_backward_workspace_size",
           "pkm_memplus_backward", "pkm_qproj_workspace_size", "pkm_qproj_forward",
           "pkm_qproj_backward", "pkm_sparse_optimizer_step", "pkm_engram_forward",
           "pkm_select", "embbag_forward_range", "pkm_check_wait_timeout")

_lib = None


def load(path: str = LIB_PATH):
    """Load libpkm.so and declare its signatures (raises if it is missing)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libpkm.so not built at {path}; run python -m sparse_key_value_b200.build")
    lib = ctypes.CDLL(path)
    FA, BA = ctypes.POINTER(FwdArgs), ctypes.POINTER(BwdArgs)
    lib.pkm_forward_workspace_size.argtypes = [FA]
    lib.pkm_forward_workspace_size.restype = SZ
    lib.pkm_check_wait_timeout.argtypes = [I64, P, P]
    lib.pkm_check_wait_timeout.restype = ctypes.c_int
    lib.pkm_select.argtypes = [FA, P]
    lib.pkm_select.restype = ctypes.c_int
    lib.embbag_forward_range.argtypes = [P, I64, I64, I32, ctypes.c_int, P, P, I64, I32, P, P]
    lib.embbag_forward_range.restype = ctypes.c_int
    lib.pkm_forward.argtypes = [FA, P]
    lib.pkm_forward.restype = ctypes.c_int
    lib.pkm_backward_workspace_size.argtypes = [BA]
    lib.pkm_backward_workspace_size.restype = SZ
    lib.pkm_backward.argtypes = [BA, P]
    lib.pkm_backward.restype = ctypes.c_int
    lib.embbag_forward.argtypes = [P, I64, I32, ctypes.c_int, P, P, I64, I32, P, P, P]
    lib.embbag_forward.restype = ctypes.c_int
    lib.embbag_backward_workspace_size.argtypes = [I64, I32, I32, I64]
    lib.embbag_backward_workspace_size.restype = SZ
    lib.embbag_backward.argtypes = [P, P, P, I64, I32, I32, ctypes.c_int, P, I64, P, P, P, P,
                                    I64, P, P, SZ, P]
    lib.embbag_backward.restype = ctypes.c_int
    lib.pkm_get_device_error.argtypes = [P, ctypes.POINTER(I32)]
    lib.pkm_get_device_error.restype = ctypes.c_int
    lib.pkm_status_string.argtypes = [ctypes.c_int]
    lib.pkm_status_string.restype = ctypes.c_char_p
    lib.pkm_version.argtypes = []
    lib.pkm_version.restype = I32
    lib.pkm_forward_noalloc.argtypes = [FA, P]
    lib.pkm_forward_noalloc.restype = ctypes.c_int
    lib.pkm_launch_count.argtypes = []
    lib.pkm_launch_count.restype = ctypes.c_uint64
    MA, QA = ctypes.POINTER(MemplusBwdArgs), ctypes.POINTER(QprojArgs)
    lib.pkm_memplus_backward_workspace_size.argtypes = [MA]
    lib.pkm_memplus_backward_workspace_size.restype = SZ
    lib.pkm_memplus_backward.argtypes = [MA, P]
    lib.pkm_memplus_backward.restype = ctypes.c_int
    lib.pkm_qproj_workspace_size.argtypes = [QA]
    lib.pkm_qproj_workspace_size.restype = SZ
    lib.pkm_qproj_forward.argtypes = [QA, P]
    lib.pkm_qproj_forward.restype = ctypes.c_int
    lib.pkm_qproj_backward.argtypes = [QA, P]
    lib.pkm_qproj_backward.restype = ctypes.c_int
    lib.pkm_engram_forward.argtypes = [ctypes.POINTER(EngramArgs), P]
    lib.pkm_engram_forward.restype = ctypes.c_int
    lib.pkm_sparse_optimizer_step.argtypes = [ctypes.POINTER(SparseOptArgs), P]
    lib.pkm_sparse_optimizer_step.restype = ctypes.c_int
    if path == LIB_PATH:
        _lib = lib
    return lib


def check(code: int, what: str):
    if code != PKM_OK:
        raise PKMError(code, what)
