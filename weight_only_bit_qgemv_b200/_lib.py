"""ctypes declarations of libwoq's C ABI (include/woq.h). No compute happens here."""

from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwoq.so")

WOQ_OK = 0
WOQ_EINVAL = -1
WOQ_ESHAPE = -2
WOQ_EALIGN = -3
WOQ_ERANGE = -4
WOQ_EDEVICE = -5
WOQ_ECUDA = -6
WOQ_ETIMEOUT = -7
WOQ_EWORKSPACE = -8

WOQ_PATH_AUTO = 0
WOQ_PATH_FP32 = 1
WOQ_PATH_BF16_TC = 2
WOQ_PATH_SPLIT_TC = 3
WOQ_GEMV_AUTO = 0
WOQ_GEMV_CUDA_CORE = 1
WOQ_GEMV_SPLIT_TC = 2
WOQ_GEMV_SPLIT_GEMM = 3
WOQ_GEMV_INT8_TC = 4
WOQ_EPI_NONE = 0
WOQ_EPI_SWIGLU = 1
WOQ_EPI_RESIDUAL = 2
WOQ_CHAIN_MAX_ITEMS = 8

#: Every symbol include/woq.h declares.
EXPORTS = (
    "qpack",
    "qgemv",
    "qgemv_path",
    "qgemv_swiglu",
    "qgemv_residual",
    "qgemv_argmax",
    "qgemv_chain_workspace_bytes",
    "qgemv_chain",
    "qgemm_workspace_bytes",
    "qgemm",
    "qgemm_bf16_noalloc",
    "woq_device_status",
    "woq_debug_set_wait_limit",
    "woq_status_str",
    "woq_launch_count",
    "woq_abi_version",
)


class WoqWeight(ctypes.Structure):
    _fields_ = [
        ("bits", ctypes.c_int32),
        ("block", ctypes.c_int32),
        ("n", ctypes.c_int64),
        ("k", ctypes.c_int64),
        ("packed", ctypes.c_void_p),
        ("scales", ctypes.c_void_p),
    ]


class WoqChainItem(ctypes.Structure):
    _fields_ = [
        ("w", ctypes.POINTER(WoqWeight)),
        ("x", ctypes.c_void_p),
        ("y", ctypes.c_void_p),
        ("r", ctypes.c_void_p),
        ("epilogue", ctypes.c_int32),
    ]


class WoqError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_str(status)} ({status})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if libwoq.so has not been built (no fallback exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"libwoq.so not found at {LIB_PATH}; build it with "
            "`python -m weight_only_bit_qgemv_b200.build` (there is no CPU fallback)"
        )
    L = ctypes.CDLL(LIB_PATH)
    c_i64, c_i32, vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p
    wp = ctypes.POINTER(WoqWeight)
    L.qpack.argtypes = [vp, c_i64, c_i64, c_i32, vp, vp]
    L.qpack.restype = ctypes.c_int
    L.qgemv.argtypes = [vp, c_i64, wp, vp, vp]
    L.qgemv.restype = ctypes.c_int
    L.qgemv_path.argtypes = [vp, c_i64, wp, vp, c_i32, vp]
    L.qgemv_path.restype = ctypes.c_int
    L.qgemv_swiglu.argtypes = [vp, c_i64, wp, vp, vp]
    L.qgemv_swiglu.restype = ctypes.c_int
    L.qgemv_residual.argtypes = [vp, c_i64, wp, vp, vp, vp]
    L.qgemv_residual.restype = ctypes.c_int
    L.qgemv_argmax.argtypes = [vp, c_i64, wp, vp, vp, vp]
    L.qgemv_argmax.restype = ctypes.c_int
    L.qgemv_chain_workspace_bytes.argtypes = []
    L.qgemv_chain_workspace_bytes.restype = ctypes.c_size_t
    L.qgemv_chain.argtypes = [ctypes.POINTER(WoqChainItem), c_i32, c_i64, vp, ctypes.c_size_t, vp]
    L.qgemv_chain.restype = ctypes.c_int
    L.qgemm_workspace_bytes.argtypes = [c_i64, wp, c_i32]
    L.qgemm_workspace_bytes.restype = ctypes.c_size_t
    L.qgemm.argtypes = [vp, c_i64, wp, vp, c_i32, vp, ctypes.c_size_t, vp]
    L.qgemm.restype = ctypes.c_int
    L.qgemm_bf16_noalloc.argtypes = [vp, c_i64, wp, vp, vp]
    L.qgemm_bf16_noalloc.restype = ctypes.c_int
    L.woq_device_status.argtypes = [ctypes.c_int]
    L.woq_device_status.restype = ctypes.c_int
    L.woq_debug_set_wait_limit.argtypes = [ctypes.c_longlong]
    L.woq_debug_set_wait_limit.restype = None
    L.woq_status_str.argtypes = [ctypes.c_int]
    L.woq_status_str.restype = ctypes.c_char_p
    L.woq_launch_count.argtypes = []
    L.woq_launch_count.restype = ctypes.c_uint64
    L.woq_abi_version.argtypes = []
    L.woq_abi_version.restype = ctypes.c_int
    _lib = L
    return L


def status_str(status: int) -> str:
    return lib().woq_status_str(status).decode()


def check(status: int, what: str) -> None:
    if status != WOQ_OK:
        raise WoqError(status, what)
