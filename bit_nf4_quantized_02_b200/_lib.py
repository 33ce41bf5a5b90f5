"""ctypes loader for libqlora.so (the C ABI of include/qlora.h).

Argument marshalling only.  Loading fails loudly if the library has not been
built: there is no fallback implementation.
"""

from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int, c_int64, c_size_t, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqlora.so")

QLORA_OK = 0
QLORA_ERR_INVALID_ARG = -1
QLORA_ERR_MISALIGNED = -2
QLORA_ERR_UNSUPPORTED_SHAPE = -3
QLORA_ERR_CUDA = -4
QLORA_ERR_DEVICE_TIMEOUT = -5
QLORA_ERR_WORKSPACE = -6
QLORA_ERR_SCRATCH_LIMIT = -7
QLORA_NOALLOC_MAX_NUMEL = 1 << 28
QLORA_DEFAULT_WAIT_LIMIT_NS = 4_000_000_000
QLORA_MAX_WAIT_LIMIT_NS = 60_000_000_000

QLORA_DTYPE_F32 = 0
QLORA_DTYPE_BF16 = 1
QLORA_MAX_RANK = 256

KERNEL_KINDS = {
    1: "quantize", 2: "dq_constants", 3: "dequant",
    10: "gemm_T", 11: "gemm_Y", 12: "gemm_G", 13: "gemm_dX", 14: "gemm_dL2", 15: "gemm_dL1", 16: "gemm_Z",
    17: "rank_G_dL2", 18: "rank_dL1",
    20: "splitk_finalize", 31: "fused_fwd", 40: "dropout_mask",
}


class NF4DQ(ctypes.Structure):
    """Mirror of qlora_nf4dq_t."""

    _fields_ = [
        ("n_out", c_int64),
        ("k_in", c_int64),
        ("codes", c_void_p),
        ("c2_fp8", c_void_p),
        ("c1", c_void_p),
        ("c2_mean", c_void_p),
        ("table", ctypes.c_int32),
    ]


TABLES = {"nf4": 0, "fp4": 1}   # QLORA_TABLE_NF4, QLORA_TABLE_FP4

QLORA_MAX_GROUP = 8


class FwdMember(ctypes.Structure):
    """Mirror of qlora_fwd_member_t (one linear of a grouped forward)."""

    _fields_ = [
        ("X", c_void_p),
        ("W", POINTER(NF4DQ)),
        ("L1", c_void_p),
        ("L2", c_void_p),
        ("r", ctypes.c_int32),
        ("s", c_float),
        ("Y", c_void_p),
        ("T_save", c_void_p),
    ]


class BwdMember(ctypes.Structure):
    """Mirror of qlora_bwd_member_t (one linear of a grouped backward)."""

    _fields_ = [
        ("dY", c_void_p),
        ("X", c_void_p),
        ("T_saved", c_void_p),
        ("W", POINTER(NF4DQ)),
        ("L1", c_void_p),
        ("L2", c_void_p),
        ("r", ctypes.c_int32),
        ("s", c_float),
        ("dX", c_void_p),
        ("dL1", c_void_p),
        ("dL2", c_void_p),
    ]


# name -> (restype, argtypes)
SIGNATURES = {
    "qlora_version": (c_int, []),
    "qlora_profile_start": (c_int, [c_int]),
    "qlora_profile_stop": (c_int, []),
    "qlora_profile_read": (c_int, [c_int, POINTER(c_int), POINTER(c_float)]),
    "qlora_status_str": (ctypes.c_char_p, [c_int]),
    "qlora_get_last_device_error": (c_int, [c_void_p]),
    "qlora_set_wait_limit_ns": (c_int, [ctypes.c_uint64, c_void_p]),
    "qlora_diag_expired_wait": (c_int, [c_void_p]),
    "qlora_quantize_workspace_size": (c_size_t, [c_int64]),
    "qlora_quantize_nf4_dq": (c_int, [c_void_p, c_int, c_int64, c_int64, c_void_p, c_void_p, c_void_p, c_void_p,
                                      c_void_p, c_size_t, c_void_p]),
    "qlora_quantize_4bit_dq": (c_int, [c_void_p, c_int, c_int64, c_int64, c_int, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_void_p, c_size_t, c_void_p]),
    "qlora_quantize_nf4_dq_noalloc": (c_int, [c_void_p, c_int, c_int64, c_int64, c_void_p, c_void_p, c_void_p,
                                              c_void_p, c_void_p]),
    "qlora_dequant": (c_int, [POINTER(NF4DQ), c_void_p, c_void_p]),
    "qlora_linear_fwd_workspace_size": (c_size_t, [c_int64, c_int64, c_int64, c_int]),
    "qlora_linear_bwd_workspace_size": (c_size_t, [c_int64, c_int64, c_int64, c_int]),
    "qlora_linear_fwd": (c_int, [c_void_p, c_int64, POINTER(NF4DQ), c_void_p, c_void_p, c_int, c_float, c_void_p,
                                 c_void_p, c_void_p, c_size_t, c_void_p]),
    "qlora_linear_bwd": (c_int, [c_void_p, c_void_p, c_void_p, c_int64, POINTER(NF4DQ), c_void_p, c_void_p, c_int,
                                 c_float, c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_size_t, c_void_p]),
    "qlora_linear_fwd_group_workspace_size": (c_size_t, [POINTER(FwdMember), c_int, c_int64]),
    "qlora_linear_fwd_group": (c_int, [POINTER(FwdMember), c_int, c_int64, c_void_p, c_size_t, c_void_p]),
    "qlora_linear_bwd_group_workspace_size": (c_size_t, [POINTER(BwdMember), c_int, c_int64]),
    "qlora_linear_bwd_group": (c_int, [POINTER(BwdMember), c_int, c_int64, c_int, c_void_p, c_size_t, c_void_p]),
    "qlora_linear_fwd_dropout_workspace_size": (c_size_t, [c_int64, c_int64, c_int64, c_int]),
    "qlora_linear_bwd_dropout_workspace_size": (c_size_t, [c_int64, c_int64, c_int64, c_int]),
    "qlora_linear_fwd_dropout": (c_int, [c_void_p, c_int64, POINTER(NF4DQ), c_void_p, c_void_p, c_int, c_float,
                                         c_void_p, c_float, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                         c_void_p]),
    "qlora_linear_bwd_dropout": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int64, POINTER(NF4DQ), c_void_p,
                                         c_void_p, c_int, c_float, c_void_p, c_float, c_void_p, c_void_p, c_void_p,
                                         c_int, c_void_p, c_size_t, c_void_p]),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load libqlora.so (once) and declare every entry point's signature."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"libqlora.so is not built ({LIB_PATH}); run `python -m bit_nf4_quantized_02_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class QLoRAError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = load()
        super().__init__(f"{where}: {lib.qlora_status_str(status).decode()} (status {status})")
        self.status = status


def check(status: int, where: str) -> None:
    if status != QLORA_OK:
        raise QLoRAError(status, where)
