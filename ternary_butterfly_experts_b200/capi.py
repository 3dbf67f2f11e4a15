"""ctypes binding of libbfmoe.so (include/bfmoe.h).

Argument marshalling only: every step of the forward runs in the library's
CUDA kernels.  Loading fails loudly when the library is missing; there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbfmoe.so")
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "bfmoe.h")

BFMOE_OK = 0
BFMOE_EINVAL = 1
BFMOE_ENOT_TERNARY = 2
BFMOE_EUNSUPPORTED = 3
BFMOE_EWORKSPACE = 4
BFMOE_ECUDA = 5
BFMOE_EDEVICE_TIMEOUT = 6
BFMOE_EDEVICE_BOUNDS = 7
BFMOE_F32 = 0
BFMOE_BF16 = 1
BFMOE_NOALLOC_SCRATCH_BYTES = 32 << 20

STATUS_NAMES = {0: "OK", 1: "EINVAL", 2: "ENOT_TERNARY", 3: "EUNSUPPORTED", 4: "EWORKSPACE",
                5: "ECUDA", 6: "EDEVICE_TIMEOUT", 7: "EDEVICE_BOUNDS"}


class BfmoeLayer(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("n_experts", ctypes.c_int), ("w_packed", ctypes.c_void_p),
                ("alpha", ctypes.c_float), ("theta", ctypes.c_void_p), ("phi", ctypes.c_void_p),
                ("tables", ctypes.c_void_p), ("gate_parts", ctypes.c_void_p)]


class BfmoeKernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 48), ("launches", ctypes.c_int), ("total_ms", ctypes.c_double)]


class BfmoeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"bfmoe status {status} ({STATUS_NAMES.get(status, '?')}): {msg}")
        self.status = status


_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t

SIGNATURES = {
    "bfmoe_pack_base": (_I, [_P, _I, _P, _P]),
    "bfmoe_unpack_base": (_I, [_P, _I, _P, _P]),
    "bfmoe_router_topk": (_I, [_P, _I, _I, _I, _P, _P, _I, _I, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "bfmoe_router_topk_noalloc": (_I, [_P, _I, _I, _I, _P, _P, _I, _I, _P, _P, _P, _P, _P, _P]),
    "bfmoe_forward": (_I, [ctypes.POINTER(BfmoeLayer), _P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "bfmoe_moe_forward": (_I, [ctypes.POINTER(BfmoeLayer), _P, _I, _I, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P,
                               _SZ, _P]),
    "bfmoe_moe_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "bfmoe_prepare_layer": (_I, [ctypes.POINTER(BfmoeLayer), _P, _SZ, _P]),
    "bfmoe_layer_tables_size": (_SZ, [_I, _I]),
    "bfmoe_backward": (_I, [ctypes.POINTER(BfmoeLayer), _P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                            _P, _P, _P, _SZ, _P]),
    "bfmoe_backward_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "bfmoe_moe_forward_host": (_I, [ctypes.POINTER(BfmoeLayer), _P, _I, _I, _P, _P, _I, _P, _I, _P, _SZ, _P]),
    "bfmoe_moe_host_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "bfmoe_materialize_expert": (_I, [ctypes.POINTER(BfmoeLayer), _I, _P, _P]),
    "bfmoe_decode_forward": (_I, [ctypes.POINTER(BfmoeLayer), _P, _I, _I, _I, _P, _P, _P, _P]),
    "bfmoe_prepare_gate": (_I, [_P, _I, _I, _P, _SZ, _P]),
    "bfmoe_gate_parts_size": (_SZ, [_I, _I]),
    "bfmoe_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "bfmoe_router_scratch_size": (_SZ, [_I, _I, _I, _I, _I]),
    "bfmoe_last_error": (ctypes.c_char_p, []),
    "bfmoe_check_device_error": (_I, [_P]),
    "bfmoe_launch_count": (ctypes.c_ulonglong, []),
    "bfmoe_profile_enable": (_I, [_I]),
    "bfmoe_profile_collect": (_I, [ctypes.POINTER(BfmoeKernelTime), _I, ctypes.POINTER(_I)]),
}


def header_functions() -> list:
    """Names of every function that include/bfmoe.h declares."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(bfmoe_[a-z_]+)\s*\(", text)
    return sorted(set(names))


def lib():
    """Load libbfmoe.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"{LIB_PATH} is missing: build it with "
                          "`python -m ternary_butterfly_experts_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def check(status: int) -> None:
    if status != BFMOE_OK:
        raise BfmoeError(status, lib().bfmoe_last_error().decode(errors="replace"))
