"""ctypes binding of libqlora.so: the C ABI declared in include/qlora.h.

Argument marshalling only.  Every step of the layer runs in the library's
CUDA kernels; this module hands device pointers, sizes and the current CUDA
stream across the boundary and turns status codes into exceptions.  If the
shared library has not been built the import of any entry point raises.
"""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqlora.so")

QLORA_OK = 0
STATUS_NAMES = {0: "QLORA_OK", 1: "QLORA_ERR_INVALID_ARG", 2: "QLORA_ERR_UNSUPPORTED",
                3: "QLORA_ERR_MISALIGNED", 4: "QLORA_ERR_WORKSPACE", 5: "QLORA_ERR_CUDA",
                6: "QLORA_ERR_NONFINITE", 7: "QLORA_ERR_TIMEOUT"}
OP_QUANTIZE, OP_FWD, OP_BWD = 0, 1, 2
QUANT_SNAP_DQ_SCALE = 1


class NF4Weight(C.Structure):
    """Mirror of qlora_nf4_weight."""
    _fields_ = [("codes", C.c_void_p), ("scales", C.c_void_p), ("c2", C.c_void_p),
                ("rows", C.c_int64), ("cols", C.c_int64),
                ("blocksize", C.c_int32), ("dq_block", C.c_int32),
                ("codebook", C.c_float * 16)]


class AdamHParams(C.Structure):
    """Mirror of qlora_adam_hparams."""
    _fields_ = [("lr", C.c_float), ("beta1", C.c_float), ("beta2", C.c_float), ("eps", C.c_float),
                ("weight_decay", C.c_float), ("step", C.c_int32)]


class FwdProblem(C.Structure):
    """Mirror of qlora_fwd_problem."""
    _fields_ = [("x", C.c_void_p), ("qw", C.POINTER(NF4Weight)), ("A", C.c_void_p), ("B", C.c_void_p),
                ("r", C.c_int32), ("s", C.c_float), ("y", C.c_void_p)]


class TraceRec(C.Structure):
    """Mirror of qlora_trace_rec."""
    _fields_ = [("kernel", C.c_int32), ("pad_", C.c_int32), ("start", C.c_void_p), ("stop", C.c_void_p),
                ("flops", C.c_double), ("bytes", C.c_double)]


# name -> (restype, argtypes)
SIGNATURES = {
    "qlora_status_string": (C.c_char_p, [C.c_int]),
    "qlora_version": (C.c_char_p, []),
    "qlora_nf4_codebook_eq2": (C.c_int, [C.POINTER(C.c_float)]),
    "qlora_nf4_storage_bytes": (C.c_int, [C.c_int64, C.c_int64, C.c_int32, C.c_int32,
                                          C.POINTER(C.c_size_t), C.POINTER(C.c_size_t), C.POINTER(C.c_size_t)]),
    "qlora_workspace_bytes": (C.c_size_t, [C.c_int32, C.c_int64, C.c_int64, C.c_int64, C.c_int32]),
    "qlora_workspace_init": (C.c_int, [C.c_void_p, C.c_size_t, C.c_void_p]),
    "qlora_get_error": (C.c_int, [C.c_void_p, C.c_void_p]),
    "qlora_quantize_nf4": (C.c_int, [C.c_void_p, C.c_int64, C.c_int64, C.c_int32, C.c_int32,
                                     C.POINTER(C.c_float), C.POINTER(NF4Weight), C.c_void_p, C.c_size_t,
                                     C.c_void_p]),
    "qlora_quantize_nf4_ex": (C.c_int, [C.c_void_p, C.c_int64, C.c_int64, C.c_int32, C.c_int32,
                                        C.POINTER(C.c_float), C.c_uint32, C.POINTER(NF4Weight), C.c_void_p,
                                        C.c_size_t, C.c_void_p]),
    "qlora_dequantize": (C.c_int, [C.POINTER(NF4Weight), C.c_void_p, C.c_void_p]),
    "qlora_merge_adapter": (C.c_int, [C.POINTER(NF4Weight), C.c_void_p, C.c_void_p, C.c_int32, C.c_float,
                                      C.c_void_p, C.c_void_p]),
    "qlora_linear_fwd": (C.c_int, [C.c_void_p, C.c_int64, C.POINTER(NF4Weight), C.c_void_p, C.c_void_p,
                                   C.c_int32, C.c_float, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "qlora_linear_bwd": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int64, C.POINTER(NF4Weight), C.c_void_p,
                                   C.c_void_p, C.c_int32, C.c_float, C.c_void_p, C.c_void_p, C.c_void_p,
                                   C.c_void_p, C.c_size_t, C.c_void_p]),
    "qlora_linear_fwd_noalloc": (C.c_int, [C.c_void_p, C.c_int64, C.POINTER(NF4Weight), C.c_void_p, C.c_void_p,
                                           C.c_int32, C.c_float, C.c_void_p, C.c_void_p]),
    "qlora_noalloc_get_error": (C.c_int, [C.c_void_p]),
    "qlora_decode_batch_workspace_bytes": (C.c_size_t, [C.c_int32, C.POINTER(FwdProblem), C.c_int64]),
    "qlora_linear_fwd_decode_batch": (C.c_int, [C.c_int32, C.POINTER(FwdProblem), C.c_int64, C.c_void_p,
                                                C.c_size_t, C.c_void_p]),
    "qlora_saved_u_bytes": (C.c_size_t, [C.c_int64, C.c_int32]),
    "qlora_linear_fwd_save": (C.c_int, [C.c_void_p, C.c_int64, C.POINTER(NF4Weight), C.c_void_p, C.c_void_p,
                                        C.c_int32, C.c_float, C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t,
                                        C.c_void_p]),
    "qlora_linear_bwd_saved": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int64, C.POINTER(NF4Weight), C.c_void_p,
                                         C.c_void_p, C.c_int32, C.c_float, C.c_void_p, C.c_void_p, C.c_void_p,
                                         C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "qlora_wait_selftest": (C.c_int, [C.c_void_p, C.c_size_t, C.c_uint32, C.c_void_p]),
    "qlora_adam_step": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int64,
                                  C.POINTER(AdamHParams), C.c_void_p]),
    "qlora_paged_alloc": (C.c_int, [C.c_size_t, C.POINTER(C.c_void_p)]),
    "qlora_paged_free": (C.c_int, [C.c_void_p]),
    "qlora_paged_prefetch": (C.c_int, [C.c_void_p, C.c_size_t, C.c_int32, C.c_void_p]),
    "qlora_trace_attach": (C.c_int, [C.POINTER(TraceRec), C.c_int32, C.POINTER(C.c_int32)]),
    "qlora_kernel_name": (C.c_char_p, [C.c_int32]),
}

_LIB = None


def lib() -> C.CDLL:
    """Load libqlora.so (raises if it is missing: there is no fallback)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run `python -m bit_nf4_quantized_20_b200.build`")
        handle = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = handle
    return _LIB


class QLoraError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = lib().qlora_status_string(status).decode()
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)} ({msg})")


def check(fn: str, status: int) -> None:
    if status != QLORA_OK:
        raise QLoraError(fn, status)
