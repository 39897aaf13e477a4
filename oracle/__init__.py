"""CPU oracle for weight-only block-32 int4/int8 quantised matmul.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls or links
this package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may use it. It shares no code with the CUDA library.

Everything here is plain NumPy in float64 (the one narrowing step, the scale,
is rounded once to IEEE binary16), written for a reader to check by eye
against the method's definition. See ``oracle/woq_ref.py``.

Parity pins: every function is pinned by ``tests/test_oracle.py`` to facts
fixed outside this module (closed forms, brute force, invariants, golden
fixtures under ``tests/golden/``). No function here is "parity unpinned".
"""

from .woq_ref import (  # noqa: F401
    BLOCK,
    qrange,
    int5_high_bit_position,
    row_bytes,
    fp16_round,
    fp16_bits_to_float,
    quantise,
    pack,
    unpack,
    dequantise,
    matmul_ref,
    qgemv_ref,
    qgemm_ref,
    qgemm_bf16_ref,
    greedy_ref,
    silu_ref,
    swiglu_ref,
    residual_ref,
    qgemv_argmax_ref,
    bf16_round,
)
