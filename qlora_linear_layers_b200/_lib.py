"""ctypes loader for libqlora_nf4.so: argument marshalling only.

The C ABI is declared in include/qlora_nf4.h.  This module maps each entry
point to a Python callable of the same name taking plain integers (device
addresses), sizes and stream handles.  It never computes anything itself and
has no fallback: if the library is missing, importing it raises.
"""

from __future__ import annotations

import ctypes as C
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqlora_nf4.so")

QLORA_OK = 0
QLORA_ERR_INVALID_ARG = 1
QLORA_ERR_SHAPE = 2
QLORA_ERR_ALIGN = 3
QLORA_ERR_NONFINITE = 4
QLORA_ERR_TIMEOUT = 5
QLORA_ERR_CUDA = 6
QLORA_ERR_UNSUPPORTED = 7
QLORA_ERR_WORKSPACE = 8

QLORA_F32 = 0
QLORA_BF16 = 1

QLORA_QUANT_NF4 = 0
QLORA_QUANT_FP4 = 1
QLORA_DQ_HIST_BYTES = 2048
QLORA_DQ_NONE = 0
QLORA_DQ_INT8 = 1
QLORA_DQ_FP8 = 2

QLORA_OP_DOUBLE_QUANT = 0
QLORA_OP_FWD = 1
QLORA_OP_BWD = 2
QLORA_OP_FWD_DROPOUT = 3
QLORA_OP_BWD_DROPOUT = 4

QLORA_FWD_NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024

# Every symbol the header declares, with (restype, argtypes).
_vp, _i64, _i32, _f32, _sz = C.c_void_p, C.c_int64, C.c_int, C.c_float, C.c_size_t


class NF4Weight(C.Structure):
    """Mirror of `nf4_weight` in include/qlora_nf4.h."""
    _fields_ = [
        ("packed", _vp),
        ("rows", _i64),
        ("cols", _i64),
        ("blocksize", C.c_int32),
        ("double_quant", C.c_int32),
        ("absmax", _vp),
        ("qabsmax", _vp),
        ("dq_scale", _vp),
        ("dq_mean", _vp),
        ("dq_blocksize", C.c_int32),
        ("quant_type", C.c_int32),
    ]


class Dropout(C.Structure):
    """Mirror of `qlora_dropout` in include/qlora_nf4.h."""
    _fields_ = [("p", C.c_float), ("reserved", C.c_uint32), ("seed", C.c_uint64)]


SIGNATURES = {
    "qlora_abi_version": (_i32, []),
    "qlora_kernel_launches": (C.c_uint64, []),
    "qlora_profile_gemm_events": (_i32, [_vp, _vp]),
    "qlora_status_string": (C.c_char_p, [_i32]),
    "nf4_code_table": (_i32, [C.POINTER(C.c_float)]),
    "nf4_code_thresholds": (_i32, [C.POINTER(C.c_float)]),
    "qlora_code_table": (_i32, [_i32, C.POINTER(C.c_float)]),
    "qlora_code_thresholds": (_i32, [_i32, C.POINTER(C.c_float), C.POINTER(C.c_int)]),
    "qlora_workspace_bytes": (_sz, [_i32, _i64, _i64, _i64, _i32]),
    "qlora_dq_mean_from_hist": (_i32, [C.POINTER(C.c_int64), _i64, C.POINTER(C.c_float)]),
    "nf4_quantize": (_i32, [_vp, _i32, _i64, _i64, _i32, _vp, _vp, _vp]),
    "qlora_quantize_4bit": (_i32, [_vp, _i32, _i64, _i64, _i32, _i32, _vp, _vp, _vp, _vp]),
    "nf4_double_quantize": (_i32, [_vp, _i64, _i32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "nf4_double_quantize_hist": (_i32, [_vp, _i64, _vp, _i64, _i32, _vp, _vp, _vp, _vp]),
    "qlora_double_quantize_hist": (_i32, [_vp, _i64, _vp, _i64, _i32, _i32, _vp, _vp, _vp, _vp]),
    "nf4_dequantize": (_i32, [C.POINTER(NF4Weight), _vp, _vp]),
    "qlora_merge": (_i32, [C.POINTER(NF4Weight), _vp, _vp, _i32, _f32, _vp, _vp]),
    "qlora_linear_fwd": (_i32, [C.POINTER(NF4Weight), _vp, _i64, _vp, _vp, _i32, _f32,
                                _vp, _vp, _vp, _sz, _vp]),
    "qlora_linear_bwd": (_i32, [C.POINTER(NF4Weight), _vp, _vp, _i64, _vp, _vp, _i32, _f32,
                                _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "qlora_linear_fwd_dropout": (_i32, [C.POINTER(NF4Weight), _vp, _i64, _vp, _vp, _i32, _f32,
                                        C.POINTER(Dropout), _vp, _vp, _vp, _sz, _vp]),
    "qlora_linear_bwd_dropout": (_i32, [C.POINTER(NF4Weight), _vp, _vp, _i64, _vp, _vp, _i32, _f32,
                                        C.POINTER(Dropout), _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "qlora_linear_fwd_noalloc": (_i32, [C.POINTER(NF4Weight), _vp, _i64, _vp, _vp, _i32, _f32,
                                        _vp, _vp, _vp]),
    "qlora_check_status": (_i32, [_vp]),
    "qlora_set_wait_limit": (_i32, [C.c_uint64]),
    "qlora_test_withhold_first_fill": (_i32, [_i32]),
}

_lib = None


def load() -> C.CDLL:
    """Load the in-tree library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m qlora_linear_layers_b200.build`")
        lib = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class QLoraError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = load().qlora_status_string(code).decode()
        super().__init__(f"{where}: {msg} (status {code})")


def check(code: int, where: str) -> None:
    if code != QLORA_OK:
        raise QLoraError(code, where)
