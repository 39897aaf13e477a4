"""Plain, slow, obviously correct CPU definition of weight-only block-32 qgemv/qgemm.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``). The CUDA library never
imports this file and this file imports nothing from the library.

What the method computes, and where it is stated:

* "TinyMOSS-Diarize" (devpost), section "How we built it": the kernels are
  weight-only; activations stay FP32; dequantisation is fused into the matmul
  and no dequantised weight tensor is ever materialised; the packed tensors
  live in a container with a 64-byte-aligned tensor table.
* "MOSS-Transcribe-Diarize -- LiteRT (TFLite)", section "Files" (production
  set) and "v2 decoder": the production decoder is "q4b32", int4 in blocks of
  32 values.
* "MOSS Transcribe Diarize 0.9B" (soniqo, Russian guide), section
  "Implementation notes": the decoder uses symmetric linear INT8 quantisation
  with block 32.
* "MOSS Transcribe Diarize 0.9B" (soniqo, English guide), section "INT5 vs
  INT8": the decoder is also deployed with 5-bit weights (the pages give no
  5-bit layout; the one below is this library's).

Readings where the pages are silent (each listed in the design notes):

* the scale of a block is max|w| / qmax with qmax = 2^(bits-1) - 1 (7 or 127),
  computed in float64 and rounded ONCE, round-half-even, to IEEE binary16;
  a scale that rounds to +inf is an error; subnormal binary16 scales are kept;
* codes are computed against the STORED binary16 scale:
  q = clamp(round_half_even(w / s), qmin, qmax) in float64, qmin = -2^(bits-1);
  an all-zero (or underflowed, s == 0) block gets q = 0 everywhere;
* packing: int4 byte j of a row holds element 2j in bits 0-3 and element
  2j+1 in bits 4-7, 4-bit two's complement; int8 is one two's-complement byte
  per element; int5 (codes -16..15, 5-bit two's complement) stores a row as
  K/2 bytes holding the low four bits of every code laid out as int4, then
  one little-endian 32-bit word per block holding bit 4 of every code of the
  block, element e of the block at bit e//8 + 4*(e%4) + 16*((e%8)//4);
  scales are binary16 bit patterns in a separate [N, K/32] array;
* W is [N, K] (out, in) and Y = X . W^T, exactly, in float64.

Nothing here is blocked, fused or reordered: each function is one step of the
definition above, written out.
"""

from __future__ import annotations

import math

import numpy as np

BLOCK = 32


def qrange(bits: int) -> tuple[int, int]:
    """(qmin, qmax) of symmetric signed ``bits``-bit codes: (-8, 7), (-16, 15) or (-128, 127)."""
    if bits not in (4, 5, 8):
        raise ValueError(f"bits must be 4, 5 or 8, got {bits}")
    return -(1 << (bits - 1)), (1 << (bits - 1)) - 1


def int5_high_bit_position(e: int) -> int:
    """Bit of a block's 32-bit high-bit word that holds bit 4 of the block's element e."""
    return e // 8 + 4 * (e % 4) + 16 * ((e % 8) // 4)


def row_bytes(K: int, bits: int) -> int:
    """Bytes of one packed row of K codes."""
    return K * bits // 8


def fp16_round(v: np.ndarray) -> np.ndarray:
    """Round float64 values once, half-to-even, to binary16; return the bit patterns.

    NumPy converts float64 to float16 directly from the double's bits (one
    rounding), which is the reading taken for the block scale. Raises
    ``OverflowError`` if any value rounds to infinity.
    """
    v = np.asarray(v, dtype=np.float64)
    with np.errstate(over="ignore"):
        h = v.astype(np.float16)
    if not np.all(np.isfinite(h)):
        raise OverflowError("block scale overflows binary16")
    return h.view(np.uint16)


def fp16_bits_to_float(bits: np.ndarray) -> np.ndarray:
    """Exact float64 value of binary16 bit patterns."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def quantise(W: np.ndarray, bits: int) -> tuple[np.ndarray, np.ndarray]:
    """Symmetric block-32 quantisation of W [N, K] float32 along K.

    Returns (q, scale_bits): q int32 [N, K] in [qmin, qmax], scale_bits uint16
    [N, K/32] binary16 patterns. Steps, per row n and block j:
      1. a = max |W[n, 32j:32j+32]|   (exact, over the float32 values)
      2. s = fp16_RNE(float64(a) / qmax)
      3. q = clamp(rint_half_even(float64(w) / float64(s)), qmin, qmax), or 0 if s == 0
    """
    W = np.asarray(W)
    if W.dtype != np.float32:
        raise TypeError("W must be float32")
    if W.ndim != 2:
        raise ValueError("W must be 2-D [N, K]")
    N, K = W.shape
    if N <= 0 or K <= 0 or K % BLOCK != 0:
        raise ValueError(f"K must be a positive multiple of {BLOCK}, got {K}")
    if not np.all(np.isfinite(W)):
        raise ValueError("W has non-finite values")
    qmin, qmax = qrange(bits)
    blocks = W.astype(np.float64).reshape(N, K // BLOCK, BLOCK)
    a = np.max(np.abs(blocks), axis=2)                      # step 1
    scale_bits = fp16_round(a / float(qmax))                # step 2
    s = fp16_bits_to_float(scale_bits)[:, :, None]
    q = np.zeros_like(blocks)
    nz = np.broadcast_to(s != 0.0, blocks.shape)
    q[nz] = np.rint(blocks[nz] / np.broadcast_to(s, blocks.shape)[nz])   # step 3
    q = np.clip(q, qmin, qmax)
    return q.reshape(N, K).astype(np.int32), scale_bits


def pack(q: np.ndarray, bits: int) -> np.ndarray:
    """Pack codes q [N, K] into bytes [N, K*bits/8] (layout in the module docstring)."""
    q = np.asarray(q)
    qmin, qmax = qrange(bits)
    if q.min(initial=0) < qmin or q.max(initial=0) > qmax:
        raise ValueError("code out of range")
    N, K = q.shape
    if bits == 8:
        return q.astype(np.int8).view(np.uint8).reshape(N, K).copy()
    if bits == 5:
        u = q.astype(np.int64) & 0x1F                       # 5-bit two's complement
        nibbles = pack(((u & 0xF) ^ 8) - 8, 4)              # low four bits, laid out as int4
        high = np.zeros((N, K // BLOCK), dtype=np.uint32)
        for e in range(BLOCK):                              # bit 4 of element e of each block
            bit4 = ((u[:, e::BLOCK] >> 4) & 1).astype(np.uint32)
            high |= bit4 << np.uint32(int5_high_bit_position(e))
        return np.concatenate([nibbles, high.astype("<u4").view(np.uint8)], axis=1)
    u = (q.astype(np.int64) & 0xF).astype(np.uint8)        # 4-bit two's complement
    lo = u[:, 0::2]                                         # element 2j -> bits 0-3
    hi = u[:, 1::2]                                         # element 2j+1 -> bits 4-7
    return (lo | (hi << 4)).astype(np.uint8)


def unpack(packed: np.ndarray, bits: int, K: int) -> np.ndarray:
    """Inverse of ``pack``: bytes [N, K*bits/8] -> codes int32 [N, K] (all 2^bits codes)."""
    packed = np.asarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    if bits == 8:
        return packed.view(np.int8).astype(np.int32).reshape(N, K)
    if bits == 5:
        low = unpack(packed[:, :K // 2], 4, K) & 0xF                 # low four bits
        high = np.ascontiguousarray(packed[:, K // 2:]).view("<u4").astype(np.int64)
        u = np.empty((N, K), dtype=np.int64)
        for e in range(BLOCK):
            bit4 = (high >> int5_high_bit_position(e)) & 1
            u[:, e::BLOCK] = low[:, e::BLOCK] | (bit4 << 4)
        return np.where(u >= 16, u - 32, u).astype(np.int32)
    lo = (packed & 0xF).astype(np.int32)
    hi = (packed >> 4).astype(np.int32)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    q = np.empty((N, K), dtype=np.int32)
    q[:, 0::2] = lo
    q[:, 1::2] = hi
    return q


def dequantise(q: np.ndarray, scale_bits: np.ndarray) -> np.ndarray:
    """W_hat[n, k] = float64(s[n, k // 32]) * q[n, k]  (exact in float64)."""
    q = np.asarray(q)
    N, K = q.shape
    s = fp16_bits_to_float(scale_bits)
    if s.shape != (N, K // BLOCK):
        raise ValueError("scale array has the wrong shape")
    return q.astype(np.float64) * np.repeat(s, BLOCK, axis=1)


def matmul_ref(X: np.ndarray, W_hat: np.ndarray) -> np.ndarray:
    """Y = X . W_hat^T in float64 (X [M, K] taken exactly from float32)."""
    X = np.asarray(X, dtype=np.float64)
    return X @ np.asarray(W_hat, dtype=np.float64).T


def qgemv_ref(X: np.ndarray, packed: np.ndarray, scale_bits: np.ndarray, bits: int) -> np.ndarray:
    """Reference for the FP32 paths: unpack, dequantise, multiply, all in float64."""
    X = np.atleast_2d(np.asarray(X))
    K = X.shape[1]
    q = unpack(packed, bits, K)
    return matmul_ref(X, dequantise(q, scale_bits))


qgemm_ref = qgemv_ref


def bf16_round(v: np.ndarray) -> np.ndarray:
    """Round float64 values once, half-to-even, to bfloat16 (8 significant bits).

    Valid for finite values whose magnitude is 0 or in bfloat16's normal
    range [2^-126, 2^128); returns float64.
    """
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)                 # v = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def qgemm_bf16_ref(X: np.ndarray, packed: np.ndarray, scale_bits: np.ndarray, bits: int) -> np.ndarray:
    """The bf16 tensor-core reading: Y = bf16(X) . bf16(s*q)^T with exact accumulation.

    Reading taken: X is rounded once to bf16; each dequantised weight s*q (exact
    in float32) is rounded once to bf16; products are summed exactly (float64).
    The exact ``qgemm_ref`` stays the acceptance reference; this one measures
    how far a kernel is from the roundings it claims to make.
    """
    X = np.atleast_2d(np.asarray(X, dtype=np.float64))
    K = X.shape[1]
    W_hat = dequantise(unpack(packed, bits, K), scale_bits)
    return matmul_ref(bf16_round(X), bf16_round(W_hat))


def silu_ref(g: np.ndarray) -> np.ndarray:
    """SiLU, g * sigmoid(g) = g / (1 + exp(-g)), in float64 (written as g * sigmoid for large
    negative g, where exp(-g) overflows)."""
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(over="ignore"):
        return np.where(g >= 0, g / (1.0 + np.exp(-g)), g * np.exp(g) / (1.0 + np.exp(g)))


def swiglu_ref(X: np.ndarray, packed: np.ndarray, scale_bits: np.ndarray, bits: int) -> np.ndarray:
    """SwiGLU over a row-interleaved gate|up weight: Y = qgemv_ref(...), then
    silu(Y[:, 0::2]) * Y[:, 1::2] in float64."""
    Y = qgemv_ref(X, packed, scale_bits, bits)
    return silu_ref(Y[:, 0::2]) * Y[:, 1::2]


def residual_ref(X: np.ndarray, packed: np.ndarray, scale_bits: np.ndarray, bits: int,
                 R: np.ndarray) -> np.ndarray:
    """A projection added to the residual stream: qgemv_ref(X, ...) + R in float64. The text
    backbone is a Qwen3-0.6B-style causal decoder (evermx article on MOSS-Transcribe-Diarize,
    "Architecture"; LiteRT model card, "Files": Qwen3-0.6B blocks), a pre-norm transformer
    whose attention output projection and MLP down projection are each added to the hidden
    state they were computed from."""
    return qgemv_ref(X, packed, scale_bits, bits) + np.asarray(R, dtype=np.float64)


def greedy_ref(Y: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Greedy decoding's pick over each row of outputs Y [M, N]: the first index of the
    row maximum, and that maximum ("MOSS Transcribe Diarize 0.9B", soniqo Russian guide,
    "Implementation notes": the runtime decodes greedily). NaN counts as the maximum.
    """
    Y = np.atleast_2d(np.asarray(Y, dtype=np.float64))
    idx = np.empty(Y.shape[0], dtype=np.int64)
    for i, row in enumerate(Y):
        nan = np.flatnonzero(np.isnan(row))
        idx[i] = nan[0] if nan.size else int(np.argmax(row))
    return idx, Y[np.arange(Y.shape[0]), idx]


def qgemv_argmax_ref(X: np.ndarray, packed: np.ndarray, scale_bits: np.ndarray, bits: int):
    """Greedy pick over the exact outputs: greedy_ref(qgemv_ref(...))."""
    return greedy_ref(qgemv_ref(X, packed, scale_bits, bits))


def fsum_dot(x_row: np.ndarray, w_row: np.ndarray) -> float:
    """Correctly rounded dot product of two float64 vectors (math.fsum), for tiny cases."""
    return math.fsum(float(a) * float(b) for a, b in zip(x_row, w_row))
