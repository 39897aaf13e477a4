"""Weight-only block-32 int4/int8 qgemv/qgemm for B200 (sm_100a).

Thin Python binding over libwoq's C ABI (include/woq.h). PyTorch provides device memory
and streams only; every step of the computation runs in the library's CUDA kernels (or,
for ``qpack``, in its host C++ quantiser). There is no CPU or PyTorch fallback: if the
library is missing, every call raises.

    w = pack(W_fp32_cpu, bits=4, device="cuda")    # qpack on the host, copy to HBM
    y = qgemv(x, w)                                # decode, 1 <= m <= 64, FP32
    Y = qgemm(X, w, path="bf16_tc")                # prefill, tcgen05 tensor cores
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import (  # noqa: F401
    WOQ_GEMV_AUTO,
    WOQ_GEMV_CUDA_CORE,
    WOQ_GEMV_SPLIT_TC,
    WOQ_GEMV_SPLIT_GEMM,
    WOQ_GEMV_INT8_TC,
    WOQ_PATH_AUTO,
    WOQ_PATH_BF16_TC,
    WOQ_PATH_FP32,
    WOQ_PATH_SPLIT_TC,
    WoqError,
)

__all__ = [
    "PackedWeight",
    "qpack",
    "pack",
    "qgemv",
    "qgemv_argmax",
    "qgemv_swiglu",
    "qgemv_residual",
    "interleave_rows",
    "ChainItem",
    "chain_workspace",
    "qgemv_chain",
    "qgemm",
    "qgemm_workspace_bytes",
    "qgemm_bf16_noalloc",
    "device_status",
    "launch_count",
    "WoqError",
]

_PATHS = {
    "auto": WOQ_PATH_AUTO,
    "fp32": WOQ_PATH_FP32,
    "bf16_tc": WOQ_PATH_BF16_TC,
    "split_tc": WOQ_PATH_SPLIT_TC,
}
_GEMV_PATHS = {
    "auto": WOQ_GEMV_AUTO,
    "cuda_core": WOQ_GEMV_CUDA_CORE,
    "split_tc": WOQ_GEMV_SPLIT_TC,
    "split_gemm": WOQ_GEMV_SPLIT_GEMM,
    "int8_tc": WOQ_GEMV_INT8_TC,
}


def _ptr(t: torch.Tensor) -> int:
    return t.data_ptr()


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


@dataclass
class PackedWeight:
    """One packed weight in device memory, in the layout of include/woq.h."""

    packed: torch.Tensor  # uint8 [n, k*bits/8]
    scales: torch.Tensor  # int16 [n, k/32], binary16 bit patterns
    bits: int
    n: int
    k: int

    def desc(self) -> _lib.WoqWeight:
        return _lib.WoqWeight(self.bits, 32, self.n, self.k, _ptr(self.packed), _ptr(self.scales))

    @property
    def nbytes(self) -> int:
        """Packed codes plus scales: the bytes one product streams from memory."""
        return self.packed.numel() + 2 * self.scales.numel()

    def to(self, device) -> "PackedWeight":
        return PackedWeight(self.packed.to(device), self.scales.to(device), self.bits, self.n, self.k)


def qpack(W: torch.Tensor, bits: int) -> tuple[torch.Tensor, torch.Tensor]:
    """Host quantiser (C ABI ``qpack``): W float32 [n, k] on the CPU -> (packed, scales);
    bits 4, 5 or 8 (layouts in include/woq.h)."""
    if W.device.type != "cpu" or W.dtype != torch.float32 or W.dim() != 2:
        raise ValueError("qpack takes a 2-D float32 CPU tensor")
    W = W.contiguous()
    n, k = W.shape
    if bits not in (4, 5, 8) or k % 32:
        raise ValueError("bits must be 4, 5 or 8 and k a multiple of 32")
    packed = torch.empty(n, k * bits // 8, dtype=torch.uint8)
    scales = torch.empty(n, k // 32, dtype=torch.int16)
    _lib.check(_lib.lib().qpack(_ptr(W), n, k, bits, _ptr(packed), _ptr(scales)), "qpack")
    return packed, scales


def pack(W: torch.Tensor, bits: int, device="cuda") -> PackedWeight:
    """qpack on the host, then one copy of codes and scales to ``device``."""
    packed, scales = qpack(W, bits)
    n, k = W.shape
    return PackedWeight(packed.to(device), scales.to(device), bits, n, k)


def qgemv(
    x: torch.Tensor,
    w: PackedWeight,
    out: torch.Tensor | None = None,
    stream=None,
    path: str = "auto",
) -> torch.Tensor:
    """y[m, n] = x[m, k] . W_hat^T, 1 <= m <= 64, FP32 accuracy (C ABI ``qgemv_path``);
    path in {"auto", "cuda_core", "split_tc", "split_gemm", "int8_tc"}."""
    if x.dtype != torch.float32 or not x.is_cuda or x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous 2-D float32 CUDA tensor")
    m = x.shape[0]
    if out is None:
        out = torch.empty(m, w.n, dtype=torch.float32, device=x.device)
    d = w.desc()
    rc = _lib.lib().qgemv_path(_ptr(x), m, ctypes.byref(d), _ptr(out), _GEMV_PATHS[path], _stream(stream))
    _lib.check(rc, "qgemv")
    return out


def interleave_rows(W_gate: torch.Tensor, W_up: torch.Tensor) -> torch.Tensor:
    """[I, k] gate and up weights -> [2I, k] with row 2i = gate i, row 2i+1 = up i, the
    layout qgemv_swiglu expects."""
    if W_gate.shape != W_up.shape:
        raise ValueError("gate and up weights must have the same shape")
    return torch.stack([W_gate, W_up], dim=1).reshape(2 * W_gate.shape[0], W_gate.shape[1])


def qgemv_swiglu(x: torch.Tensor, w: PackedWeight, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y[m, n/2] = silu(gate) * up over a row-interleaved gate|up weight (C ABI ``qgemv_swiglu``)."""
    if x.dtype != torch.float32 or not x.is_cuda or x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous 2-D float32 CUDA tensor")
    m = x.shape[0]
    if out is None:
        out = torch.empty(m, w.n // 2, dtype=torch.float32, device=x.device)
    d = w.desc()
    _lib.check(_lib.lib().qgemv_swiglu(_ptr(x), m, ctypes.byref(d), _ptr(out), _stream(stream)), "qgemv_swiglu")
    return out


def qgemv_argmax(x: torch.Tensor, w: PackedWeight, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Per activation row, the index (smallest among ties) and value of the largest output of
    x . W_hat^T, without writing the outputs (C ABI ``qgemv_argmax``); 1 <= m <= 8."""
    if x.dtype != torch.float32 or not x.is_cuda or x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous 2-D float32 CUDA tensor")
    m = x.shape[0]
    idx = torch.empty(m, dtype=torch.int64, device=x.device)
    val = torch.empty(m, dtype=torch.float32, device=x.device)
    d = w.desc()
    rc = _lib.lib().qgemv_argmax(_ptr(x), m, ctypes.byref(d), _ptr(idx), _ptr(val), _stream(stream))
    _lib.check(rc, "qgemv_argmax")
    return idx, val


def qgemv_residual(x: torch.Tensor, w: PackedWeight, r: torch.Tensor, out: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """y = x . W_hat^T + r with the add fused (C ABI ``qgemv_residual``); ``out`` may be ``r``
    for an in-place update of the residual stream."""
    if x.dtype != torch.float32 or not x.is_cuda or x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous 2-D float32 CUDA tensor")
    m = x.shape[0]
    if r.dtype != torch.float32 or not r.is_cuda or tuple(r.shape) != (m, w.n) or not r.is_contiguous():
        raise ValueError("r must be a contiguous float32 CUDA tensor of shape [m, n]")
    if out is None:
        out = torch.empty(m, w.n, dtype=torch.float32, device=x.device)
    d = w.desc()
    rc = _lib.lib().qgemv_residual(_ptr(x), m, ctypes.byref(d), _ptr(r), _ptr(out), _stream(stream))
    _lib.check(rc, "qgemv_residual")
    return out


_EPILOGUES = {"none": _lib.WOQ_EPI_NONE, "swiglu": _lib.WOQ_EPI_SWIGLU, "residual": _lib.WOQ_EPI_RESIDUAL}


@dataclass
class ChainItem:
    """One GEMV of a qgemv_chain launch: y = x . W_hat^T, with epilogue "none", "swiglu" (rows
    interleaved gate/up; y [m, n/2]) or "residual" (y = ... + r, r may be y)."""

    w: PackedWeight
    x: torch.Tensor
    y: torch.Tensor
    r: torch.Tensor | None = None
    epilogue: str = "none"


def chain_workspace(device="cuda") -> torch.Tensor:
    """A zeroed workspace for qgemv_chain (its counters; every successful call leaves them zero)."""
    return torch.zeros(int(_lib.lib().qgemv_chain_workspace_bytes()), dtype=torch.uint8, device=device)


def qgemv_chain(items: list[ChainItem], workspace: torch.Tensor, stream=None) -> None:
    """Run the items in order as one persistent launch (C ABI ``qgemv_chain``); item i reads
    its x only after every earlier item's outputs are complete."""
    if not items:
        raise ValueError("qgemv_chain needs at least one item")
    m = items[0].x.shape[0]
    descs = [it.w.desc() for it in items]  # kept alive for the call
    arr = (_lib.WoqChainItem * len(items))()
    for i, (it, d) in enumerate(zip(items, descs)):
        for t in (it.x, it.y) + ((it.r,) if it.r is not None else ()):
            if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
                raise ValueError("chain tensors must be contiguous float32 CUDA tensors")
        if it.x.shape[0] != m:
            raise ValueError("every item must have the same number of activation rows")
        arr[i].w = ctypes.pointer(d)
        arr[i].x = _ptr(it.x)
        arr[i].y = _ptr(it.y)
        arr[i].r = _ptr(it.r) if it.r is not None else None
        arr[i].epilogue = _EPILOGUES[it.epilogue]
    rc = _lib.lib().qgemv_chain(arr, len(items), m, _ptr(workspace), workspace.numel(), _stream(stream))
    _lib.check(rc, "qgemv_chain")


def qgemm_workspace_bytes(m: int, w: PackedWeight, path: str = "auto") -> int:
    d = w.desc()
    return int(_lib.lib().qgemm_workspace_bytes(m, ctypes.byref(d), _PATHS[path]))


def qgemm(
    X: torch.Tensor,
    w: PackedWeight,
    path: str = "auto",
    out: torch.Tensor | None = None,
    workspace: torch.Tensor | None = None,
    stream=None,
) -> torch.Tensor:
    """Y[m, n] = X[m, k] . W_hat^T (C ABI ``qgemm``); path in {"auto", "fp32", "bf16_tc", "split_tc"}."""
    if X.dtype != torch.float32 or not X.is_cuda or X.dim() != 2 or not X.is_contiguous():
        raise ValueError("X must be a contiguous 2-D float32 CUDA tensor")
    m = X.shape[0]
    p = _PATHS[path]
    if out is None:
        out = torch.empty(m, w.n, dtype=torch.float32, device=X.device)
    d = w.desc()
    need = int(_lib.lib().qgemm_workspace_bytes(m, ctypes.byref(d), p))
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    ws_ptr = _ptr(workspace) if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _lib.check(
        _lib.lib().qgemm(_ptr(X), m, ctypes.byref(d), _ptr(out), p, ws_ptr, ws_bytes, _stream(stream)),
        "qgemm",
    )
    return out


def qgemm_bf16_noalloc(X: torch.Tensor, w: PackedWeight, out: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """The bf16 tensor-core qgemm with no workspace and no device allocation in the library
    (C ABI ``qgemm_bf16_noalloc``): the bf16 copy of X goes to a fixed 32 MiB scratch array
    of the library's own, so m * k * 2 bytes must fit in it. ``out`` is allocated here by
    PyTorch when it is not given."""
    if X.dtype != torch.float32 or not X.is_cuda or X.dim() != 2 or not X.is_contiguous():
        raise ValueError("X must be a contiguous 2-D float32 CUDA tensor")
    m = X.shape[0]
    if out is None:
        out = torch.empty(m, w.n, dtype=torch.float32, device=X.device)
    d = w.desc()
    _lib.check(_lib.lib().qgemm_bf16_noalloc(_ptr(X), m, ctypes.byref(d), _ptr(out), _stream(stream)),
               "qgemm_bf16_noalloc")
    return out


def device_status(clear: bool = True) -> int:
    """Synchronise the device and report bounded waits that gave up (C ABI woq_device_status)."""
    return int(_lib.lib().woq_device_status(1 if clear else 0))


def launch_count() -> int:
    """Kernels the library has launched in this process."""
    return int(_lib.lib().woq_launch_count())
