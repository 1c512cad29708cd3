"""ctypes loader for libqnf4.so and the argument types of its C ABI (include/qnf4.h).

The library is built in-tree by ``bit_nf4_quantized_04_b200/build.py``. There is no
fallback: if the shared library is missing or cannot be loaded, importing this
module raises.
"""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# QNF4_LIB=checked selects the checked build (index checks in the kernels, reported as
# QNF4_ERR_BOUNDS), for tests; anything else, or unset, the library itself.
LIB_PATH = os.path.join(HERE, "libqnf4_checked.so" if os.environ.get("QNF4_LIB") == "checked"
                        else "libqnf4.so")

QNF4_OK = 0
STATUS_NAMES = {0: "OK", 1: "ERR_ARG", 2: "ERR_SHAPE", 3: "ERR_ALIGN", 4: "ERR_CUDA",
                5: "ERR_TIMEOUT", 6: "ERR_WORKSPACE", 7: "ERR_BOUNDS"}
OUT_F32, OUT_BF16 = 0, 1
OP_QUANTIZE, OP_DOUBLE_QUANT, OP_FWD, OP_BWD, OP_CHANQ_FWD, OP_CHANQ_BWD, OP_LOFTQ = 0, 1, 2, 3, 4, 5, 6
OP_LAYER_STATS, OP_QUANTIZE_WEIGHT, OP_QUANTIZE_WEIGHT_GROUP, OP_LAYER_STATS_GROUP = 7, 8, 9, 10


class Qnf4Weight(C.Structure):
    """Mirror of ``qnf4_weight``."""
    _fields_ = [("N", C.c_int64), ("K", C.c_int64), ("block1", C.c_int32), ("block2", C.c_int32),
                ("packed", C.c_void_p), ("code2", C.c_void_p), ("scale2", C.c_void_p),
                ("mean", C.c_void_p)]


P = C.c_void_p
I64 = C.c_int64
I32 = C.c_int32
F32 = C.c_float
SZ = C.c_size_t
ST = C.c_int

# name -> (restype, argtypes); every symbol include/qnf4.h declares
SIGNATURES = {
    "qnf4_nf4_codebook": (ST, [P, P]),
    "qnf4_nf4_quantize": (ST, [P, I64, I64, I32, P, P, P, P, SZ, P]),
    "qnf4_double_quant": (ST, [P, I64, I32, P, P, P, P, SZ, P]),
    "qnf4_dq_sum": (ST, [P, I64, P, P, SZ, P]),
    "qnf4_quantize_weight": (ST, [P, I64, I64, P, P, P, P, P, P, P, SZ, P]),
    "qnf4_nf4_layer_stats_group": (ST, [I32, C.POINTER(P), C.POINTER(I64), C.POINTER(I64), C.c_float,
                                        C.POINTER(P), C.POINTER(P), P, SZ, P]),
    "qnf4_quantize_weight_group": (ST, [I32, C.POINTER(P), C.POINTER(I64), C.POINTER(I64), C.POINTER(P),
                                        C.POINTER(P), C.POINTER(P), C.POINTER(P), C.POINTER(P),
                                        C.POINTER(P), P, SZ, P]),
    "qnf4_double_quant_shard": (ST, [P, I64, I32, P, I64, P, P, P, P]),
    "qnf4_dequant": (ST, [C.POINTER(Qnf4Weight), P, I32, P]),
    "qnf4_qlora_linear_fwd": (ST, [C.POINTER(Qnf4Weight), P, I64, P, P, I32, F32, P, P, SZ, P]),
    "qnf4_qlora_linear_fwd_noalloc": (ST, [C.POINTER(Qnf4Weight), P, I64, P, P, I32, F32, P, P]),
    "qnf4_qlora_linear_fwd_group": (ST, [I32, C.POINTER(Qnf4Weight), C.POINTER(P), I64, C.POINTER(P),
                                         C.POINTER(P), I32, F32, C.POINTER(P), P, SZ, P]),
    "qnf4_qlora_linear_bwd": (ST, [C.POINTER(Qnf4Weight), P, P, I64, P, P, I32, F32, P, P, P, P,
                                   SZ, P]),
    "qnf4_nf4_recon_error": (ST, [P, I64, I64, I32, P, P, SZ, P]),
    "qnf4_nf4_layer_stats": (ST, [P, I64, I64, F32, P, P, P, SZ, P]),
    "qnf4_rank_topk": (ST, [P, P, I32, I32, P]),
    "qnf4_dense_linear_fwd": (ST, [P, I64, I64, P, I64, P, P, I32, F32, P, P, SZ, P]),
    "qnf4_dense_linear_bwd": (ST, [P, I64, I64, P, P, I64, P, P, I32, F32, P, P, P, P, SZ, P]),
    "qnf4_chanq_quantize": (ST, [P, I64, I64, P, P, P, P, P, P, P]),
    "qnf4_chanq_linear_fwd": (ST, [P, P, P, P, P, P, I64, I64, P, I64, P, P, I32, F32, P, P, SZ,
                                   P]),
    "qnf4_chanq_linear_bwd": (ST, [P, P, P, P, P, P, I64, I64, P, P, I64, P, P, I32, F32, P, P,
                                   P, P, SZ, P]),
    "qnf4_chanq_learn": (ST, [P, I64, I64, I32, P, I32, P, P, P, P, P]),
    "qnf4_loftq_nf4": (ST, [P, I64, I64, I32, I32, P, P, P, P, P, P, P, P, SZ, P]),
    "qnf4_workspace_size": (SZ, [I32, I64, I64, I64, I32]),
    "qnf4_check": (ST, [P]),
    "qnf4_set_wait_timeout_ns": (ST, [C.c_uint64]),
    "qnf4_last_error": (C.c_char_p, []),
    "qnf4_launch_count": (C.c_ulonglong, []),
    "qnf4_set_timing_events": (ST, [P, P]),
}


def _load() -> C.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python bit_nf4_quantized_04_b200/build.py` "
            "(the CUDA library is required; there is no fallback)")
    lib = C.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


class Qnf4Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = lib.qnf4_last_error().decode(errors="replace")
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def call(name: str, *args) -> int:
    st = getattr(lib, name)(*args)
    if st != QNF4_OK:
        raise Qnf4Error(name, st)
    return st
