"""The C-ABI library loads and exports every symbol include/woq.h declares (CPU only).

Only calls that return before touching a device are made here: argument checks and
workspace sizing. Compute is exercised by the gpu-marked tests.
"""

import ctypes
import os
import re


from weight_only_bit_qgemv_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "woq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w \*]*?\b(\w+)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n not in ("defined",)))


def test_library_loads_and_exports_every_declared_symbol():
    L = _lib.lib()
    declared = _declared()
    assert "qpack" in declared and "qgemv" in declared and "qgemm" in declared
    assert sorted(_lib.EXPORTS) == declared
    for name in declared:
        assert hasattr(L, name), name
    assert L.woq_abi_version() == 1


def test_status_strings():
    for code in range(0, -9, -1):
        s = _lib.status_str(code)
        assert s and s != "unknown status"
    assert _lib.status_str(-99) == "unknown status"


def _w(bits=4, n=64, k=64, packed=64, scales=128, block=32):
    return _lib.WoqWeight(bits, block, n, k, packed, scales)


def test_argument_checks_return_before_touching_a_device():
    L = _lib.lib()
    ok_ptr = 1 << 20  # never dereferenced: every call below fails validation first
    cases = [
        (_w(bits=6), _lib.WOQ_EINVAL),
        (_w(bits=5, k=96), _lib.WOQ_ESHAPE),   # int5 rows must hold whole 128-code groups
        (_w(block=16), _lib.WOQ_EINVAL),
        (_w(k=48), _lib.WOQ_ESHAPE),
        (_w(n=0), _lib.WOQ_ESHAPE),
        (_w(packed=ok_ptr + 32), _lib.WOQ_EALIGN),
        (_w(scales=ok_ptr + 2), _lib.WOQ_EALIGN),
        (_w(packed=0), _lib.WOQ_EINVAL),
    ]
    for w, want in cases:
        assert L.qgemv(ok_ptr, 1, ctypes.byref(w), ok_ptr, None) == want
        assert L.qgemm(ok_ptr, 1, ctypes.byref(w), ok_ptr, 0, None, 0, None) == want
    w = _w(packed=ok_ptr, scales=ok_ptr)
    assert L.qgemv(ok_ptr, 0, ctypes.byref(w), ok_ptr, None) == _lib.WOQ_EINVAL
    assert L.qgemv(ok_ptr, 65, ctypes.byref(w), ok_ptr, None) == _lib.WOQ_EINVAL
    assert L.qgemv(None, 1, ctypes.byref(w), ok_ptr, None) == _lib.WOQ_EINVAL
    assert L.qgemv(ok_ptr + 4, 1, ctypes.byref(w), ok_ptr, None) == _lib.WOQ_EALIGN
    big = _w(k=65536, packed=ok_ptr, scales=ok_ptr)
    assert L.qgemv(ok_ptr, 1, ctypes.byref(big), ok_ptr, None) == _lib.WOQ_ESHAPE
    assert L.qgemv_path(ok_ptr, 8, ctypes.byref(w), ok_ptr, 5, None) == _lib.WOQ_EINVAL
    assert L.qgemv_path(ok_ptr, 8, ctypes.byref(w), ok_ptr, -1, None) == _lib.WOQ_EINVAL
    assert L.qgemv_path(ok_ptr, 65, ctypes.byref(w), ok_ptr, _lib.WOQ_GEMV_SPLIT_TC, None) == _lib.WOQ_EINVAL
    # qgemv_swiglu: 1 <= m <= 64, n even
    assert L.qgemv_swiglu(ok_ptr, 0, ctypes.byref(w), ok_ptr, None) == _lib.WOQ_EINVAL
    assert L.qgemv_swiglu(ok_ptr, 65, ctypes.byref(w), ok_ptr, None) == _lib.WOQ_EINVAL
    odd = _w(n=63, packed=ok_ptr, scales=ok_ptr)
    assert L.qgemv_swiglu(ok_ptr, 1, ctypes.byref(odd), ok_ptr, None) == _lib.WOQ_ESHAPE
    # qgemv_argmax: 1 <= m <= 8, k <= 8192, idx 8-byte aligned
    assert L.qgemv_argmax(ok_ptr, 0, ctypes.byref(w), ok_ptr, ok_ptr, None) == _lib.WOQ_EINVAL
    assert L.qgemv_argmax(ok_ptr, 9, ctypes.byref(w), ok_ptr, ok_ptr, None) == _lib.WOQ_EINVAL
    assert L.qgemv_argmax(ok_ptr, 1, ctypes.byref(w), None, ok_ptr, None) == _lib.WOQ_EINVAL
    assert L.qgemv_argmax(ok_ptr, 1, ctypes.byref(w), ok_ptr + 4, ok_ptr, None) == _lib.WOQ_EALIGN
    wide = _w(k=16384, packed=ok_ptr, scales=ok_ptr)
    assert L.qgemv_argmax(ok_ptr, 1, ctypes.byref(wide), ok_ptr, ok_ptr, None) == _lib.WOQ_ESHAPE
    # qgemv_residual: 1 <= m <= 64, k <= 8192, r may equal y but not overlap it otherwise
    R = L.qgemv_residual
    assert R(ok_ptr, 0, ctypes.byref(w), ok_ptr, ok_ptr, None) == _lib.WOQ_EINVAL
    assert R(ok_ptr, 65, ctypes.byref(w), ok_ptr, ok_ptr, None) == _lib.WOQ_EINVAL
    assert R(ok_ptr, 1, ctypes.byref(w), None, ok_ptr, None) == _lib.WOQ_EINVAL
    assert R(ok_ptr, 1, ctypes.byref(w), ok_ptr, None, None) == _lib.WOQ_EINVAL
    assert R(ok_ptr, 2, ctypes.byref(w), ok_ptr, ok_ptr + 4 * 64, None) == _lib.WOQ_EINVAL  # row 1 of r is row 0 of y
    assert R(ok_ptr, 1, ctypes.byref(wide), ok_ptr, ok_ptr, None) == _lib.WOQ_ESHAPE
    assert R(ok_ptr + 4, 1, ctypes.byref(w), ok_ptr, ok_ptr, None) == _lib.WOQ_EALIGN
    assert R(ok_ptr, 1, ctypes.byref(w), ok_ptr + 2, ok_ptr + 2, None) == _lib.WOQ_EALIGN
    # bf16 path: workspace checked before the device
    need = L.qgemm_workspace_bytes(256, ctypes.byref(w), _lib.WOQ_PATH_BF16_TC)
    assert need == 256 * 64 * 2
    assert L.qgemm(ok_ptr, 256, ctypes.byref(w), ok_ptr, 2, None, 0, None) == _lib.WOQ_EWORKSPACE
    assert L.qgemm(ok_ptr, 256, ctypes.byref(w), ok_ptr, 2, ok_ptr, need - 1, None) == _lib.WOQ_EWORKSPACE
    assert L.qgemm(ok_ptr, 256, ctypes.byref(w), ok_ptr, 2, ok_ptr + 16, need, None) == _lib.WOQ_EALIGN
    assert L.qgemm(ok_ptr, 4, ctypes.byref(w), ok_ptr, 7, None, 0, None) == _lib.WOQ_EINVAL


def test_workspace_sizing():
    L = _lib.lib()
    w = _w(n=1024, k=3072, packed=1 << 20, scales=1 << 20)
    assert L.qgemm_workspace_bytes(4, ctypes.byref(w), _lib.WOQ_PATH_FP32) == 0
    assert L.qgemm_workspace_bytes(4, ctypes.byref(w), _lib.WOQ_PATH_AUTO) == 0
    assert L.qgemm_workspace_bytes(23, ctypes.byref(w), _lib.WOQ_PATH_AUTO) == 0
    assert L.qgemm_workspace_bytes(127, ctypes.byref(w), _lib.WOQ_PATH_AUTO) == 0
    assert L.qgemm_workspace_bytes(512, ctypes.byref(w), _lib.WOQ_PATH_AUTO) == 512 * 3072 * 2
    assert L.qgemm_workspace_bytes(375, ctypes.byref(w), _lib.WOQ_PATH_BF16_TC) % 256 == 0
    assert L.qgemm_workspace_bytes(0, ctypes.byref(w), _lib.WOQ_PATH_BF16_TC) == 0
    assert L.qgemm_workspace_bytes(16, ctypes.byref(_w(bits=3)), 0) == 0
    # split form: X tiles written in-kernel, K-split partials summed on chip -> no workspace
    assert L.qgemm_workspace_bytes(4, ctypes.byref(w), _lib.WOQ_PATH_SPLIT_TC) == 0
    assert L.qgemm_workspace_bytes(65, ctypes.byref(w), _lib.WOQ_PATH_SPLIT_TC) == 0
    assert L.qgemm_workspace_bytes(4, ctypes.byref(w), 4) == 0


def test_launch_counter_starts_readable():
    assert _lib.lib().woq_launch_count() >= 0


def test_binding_constants_match_the_header():
    """Every integer #define of include/woq.h has the same value in the Python binding."""
    import os
    import re

    header = open(os.path.join(os.path.dirname(_lib.__file__), "..", "include", "woq.h")).read()
    defines = dict(re.findall(r"^#define (WOQ_\w+)\s+(-?\d+)\b", header, flags=re.M))
    assert len(defines) >= 17
    for name, value in defines.items():
        assert getattr(_lib, name) == int(value), name


def test_python_binding_names_every_compute_call():
    """The package exposes each compute call of the C ABI under the same name, and its
    wrappers refuse host tensors before calling into the library."""
    import pytest
    import torch

    import weight_only_bit_qgemv_b200 as woq

    for name in ("qpack", "qgemv", "qgemv_swiglu", "qgemv_residual", "qgemv_argmax", "qgemv_chain",
                 "qgemm", "qgemm_workspace_bytes", "qgemm_bf16_noalloc"):
        assert name in woq.__all__ and callable(getattr(woq, name)), name
    w = woq.PackedWeight(torch.zeros(4, 16, dtype=torch.uint8), torch.zeros(4, 1, dtype=torch.int16),
                         4, 4, 32)
    x = torch.zeros(1, 32)
    for call in (woq.qgemv, woq.qgemv_swiglu, woq.qgemv_argmax, woq.qgemm, woq.qgemm_bf16_noalloc):
        with pytest.raises(ValueError):
            call(x, w)
