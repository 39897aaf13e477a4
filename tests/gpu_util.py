"""Helpers shared by the GPU parity tests: build inputs, run the oracle, compare."""

import numpy as np
import torch

import oracle
import weight_only_bit_qgemv_b200 as woq
from weight_only_bit_qgemv_b200 import workloads

FP32_TOL = 1e-4        # max |Y - Y_ref| / max |Y_ref| for the FP32 paths
BF16_TOL = 1e-2        # ||Y - Y_ref||_F / ||Y_ref||_F for the bf16 tensor-core path
BF16_READING_TOL = 2e-5  # same, against the oracle's bf16 reading (only accumulation order differs)


def packed_from_weight(W: torch.Tensor, bits: int):
    """(device PackedWeight, host packed np.uint8, host scale bits np.uint16)."""
    p, s = woq.qpack(W, bits)
    n, k = W.shape
    pw = woq.PackedWeight(p.cuda(), s.cuda(), bits, n, k)
    return pw, p.numpy(), s.numpy().view(np.uint16)


def packed_raw(n: int, k: int, bits: int, seed: int):
    """Uniformly random codes (every code, -8 / -128 included) and random scales."""
    p, s = workloads.raw_codes(n, k, bits, seed)
    pw = woq.PackedWeight(p.cuda(), s.cuda(), bits, n, k)
    return pw, p.numpy(), s.numpy().view(np.uint16)


def max_rel(y: np.ndarray, ref: np.ndarray) -> float:
    den = np.max(np.abs(ref))
    return float(np.max(np.abs(y - ref)) / den) if den > 0 else float(np.max(np.abs(y)))


def fro_rel(y: np.ndarray, ref: np.ndarray) -> float:
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(y - ref) / den) if den > 0 else float(np.linalg.norm(y))


def ref_rows(X: np.ndarray, packed: np.ndarray, scales: np.ndarray, bits: int, rows=None):
    """Oracle output; if ``rows`` is given, only those weight rows (output columns)."""
    if rows is not None:
        packed, scales = packed[rows], scales[rows]
    return oracle.qgemv_ref(X, packed, scales, bits)


def guarded_out(m: int, n: int, pad: int = 256):
    """Output buffer with a poisoned tail that a correct kernel never writes."""
    buf = torch.full((m * n + pad,), float("nan"), dtype=torch.float32, device="cuda")
    buf[m * n:] = -12345.0
    return buf, buf[: m * n].view(m, n)


def tail_intact(buf: torch.Tensor, m: int, n: int) -> bool:
    return bool(torch.all(buf[m * n:] == -12345.0).item())
