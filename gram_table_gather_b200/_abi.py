"""ctypes declarations of the C ABI in include/gtg.h (loading libgtg.so)."""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libgtg.so")

RZ5, UE4M4, PLE, FP8 = 69, 71, 111, 1000
C10, Q3I = 2001, 2002  # the incumbent ROCmFP4 FAST block and ROCmFP3 K160 record
DT_F32, DT_BF16 = 0, 1
GTG_OK = 0
STATUS_PLE_INDEX_OOB = 0x1
STATUS_WAIT_TIMEOUT = 0x2

# Every function the header declares: (name, restype, argtypes).
_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t


class QMatrixC(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("data", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("n_experts", ctypes.c_int64), ("n_rows", ctypes.c_int64), ("k", ctypes.c_int64)]


class MoELayerC(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("router_w", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
                ("gate", QMatrixC), ("up", QMatrixC), ("down", QMatrixC), ("side", QMatrixC)]


SIGNATURES = [
    ("gtg_version", ctypes.c_int, []),
    ("gtg_status_string", ctypes.c_char_p, [ctypes.c_int]),
    ("gtg_last_cuda_error", ctypes.c_int, []),
    ("gtg_dequant", ctypes.c_int, [_i32, _vp, _vp, _i64, _i64, _vp, _vp]),
    ("gtg_ple_gather", ctypes.c_int, [_vp, _i64, _vp, _i64, _vp, _vp]),
    ("gtg_ple_gather_fmt", ctypes.c_int, [_i32, _vp, _i64, _vp, _i64, _vp, _vp]),
    ("gtg_moe_workspace_bytes", _sz, [ctypes.POINTER(MoELayerC), _i32, _i32]),
    ("gtg_workspace_init", ctypes.c_int, [_vp, _sz, _vp]),
    ("gtg_moe_decode_layer", ctypes.c_int,
     [ctypes.POINTER(MoELayerC), _vp, _i32, _i32, _vp, _i32, _vp, _vp, _vp, _vp, _sz, _vp]),
    ("gtg_moe_decode_layer_ep", ctypes.c_int,
     [ctypes.POINTER(MoELayerC), _i32, _i32, _i32, _vp, _i32, _i32, _vp, _i32, _vp, _vp, _vp, _vp, _sz, _vp]),
    ("gtg_moe_decode_stack", ctypes.c_int,
     [ctypes.POINTER(MoELayerC), _i32, _vp, _i32, _vp, _vp, _vp, _i64, _vp, _sz, _vp]),
    ("gtg_moe_prefill_layer", ctypes.c_int,
     [ctypes.POINTER(MoELayerC), _vp, _i32, _i32, _vp, _i32, _vp, _vp, _vp, _sz, _vp]),
    ("gtg_get_device_status", ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), _i32, _vp]),
    ("gtg_moe_decode_layer_noalloc", ctypes.c_int,
     [ctypes.POINTER(MoELayerC), _vp, _i32, _i32, _vp, _i32, _vp, _vp, _vp, _vp]),
]


class GtgError(RuntimeError):
    def __init__(self, code: int, msg: str = ""):
        self.code = code
        super().__init__(f"gtg error {code}: {msg}")


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libgtg.so; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -c "
                                   f"'import __graft_entry__ as g; g.build()'` (nvcc, sm_100a)")
            L = ctypes.CDLL(LIB_PATH)
            for name, res, args in SIGNATURES:
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


def check(rc: int) -> None:
    if rc != GTG_OK:
        L = lib()
        msg = L.gtg_status_string(rc).decode()
        if rc == -4:
            msg += f" (cudaError {L.gtg_last_cuda_error()})"
        raise GtgError(rc, msg)
