"""qgemm_bf16_noalloc: the tensor-core qgemm for callers that cannot allocate device memory.

Some callers can hand over inputs and outputs but cannot obtain a workspace: a plugin whose
host passes it only its tensors, a runtime that has reserved all device memory for its own
pool, or a loop that cannot afford cudaMalloc's device-wide synchronisation. The entry
point they call uses a fixed scratch array compiled into the library instead.

This file is collected last on purpose, so that a run stopping at the first failure has
already run every other test. It passes alone in a fresh process and after the others.
"""

import ctypes

import pytest
import torch

import oracle
import weight_only_bit_qgemv_b200 as woq
from weight_only_bit_qgemv_b200 import _lib, workloads
from tests.gpu_util import BF16_READING_TOL, BF16_TOL, fro_rel, packed_from_weight

pytestmark = pytest.mark.gpu


def _noalloc(X, w, Y):
    d = w.desc()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return _lib.lib().qgemm_bf16_noalloc(X.data_ptr(), X.shape[0], ctypes.byref(d), Y.data_ptr(), stream)


def test_noalloc_matches_qgemm_on_two_calls_in_a_row():
    cases = [(4, 512, 2048, 1024, 1), (8, 375, 1024, 3072, 2)]
    outs = []
    for bits, m, n, k, seed in cases:
        W = workloads.weight(n, k, seed=seed)
        w, p, s = packed_from_weight(W, bits)
        X = workloads.activations(m, k, seed=seed + 10)
        Xd = X.cuda()
        Y = torch.full((m, n), float("nan"), device="cuda")
        assert _noalloc(Xd, w, Y) == _lib.WOQ_OK
        outs.append((Xd, w, Y, X.numpy(), p, s, bits))
    torch.cuda.synchronize()
    # both calls in a row shared the scratch array; each must equal the workspace path
    for Xd, w, Y, X, p, s, bits in outs:
        Y_ref = woq.qgemm(Xd, w, path="bf16_tc")
        assert fro_rel(Y.cpu().numpy(), Y_ref.cpu().numpy()) <= BF16_READING_TOL
        assert fro_rel(Y.cpu().numpy(), oracle.qgemv_ref(X, p, s, bits)) <= BF16_TOL
    assert woq.device_status() == _lib.WOQ_OK


def test_noalloc_rejects_sizes_beyond_its_scratch():
    n, k = 64, 2048
    w, _, _ = packed_from_weight(workloads.weight(n, k, seed=3), 4)
    X = torch.zeros(16, k, device="cuda")
    Y = torch.zeros(16, n, device="cuda")
    d = w.desc()
    m_too_big = (32 << 20) // (2 * k) + 1          # bf16 copy of X would exceed 32 MiB
    rc = _lib.lib().qgemm_bf16_noalloc(X.data_ptr(), m_too_big, ctypes.byref(d), Y.data_ptr(), None)
    assert rc == _lib.WOQ_ESHAPE


def test_noalloc_allocates_nothing_and_accepts_the_exact_fit():
    """A call whose bf16 copy of X fills the 32 MiB scratch exactly is accepted and matches the
    workspace path, and a call (after a first one has loaded the library's kernels) leaves the
    device's free memory and torch's allocations unchanged."""
    n, k = 256, 2048
    W = workloads.weight(n, k, seed=21)
    w, _, _ = packed_from_weight(W, 4)
    m = (32 << 20) // (2 * k)                      # m * k * 2 == 32 MiB exactly
    X = workloads.activations(m, k, seed=22).cuda()
    Y = torch.full((m, n), float("nan"), device="cuda")
    assert _noalloc(X, w, Y) == _lib.WOQ_OK       # first call: loads modules, looks up the array
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    Y2 = torch.full((m, n), float("nan"), device="cuda")
    alloc1 = torch.cuda.memory_allocated()
    free1, _ = torch.cuda.mem_get_info()
    assert _noalloc(X, w, Y2) == _lib.WOQ_OK
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free1
    assert torch.cuda.memory_allocated() == alloc1
    assert alloc1 - alloc0 == Y2.numel() * 4 and free0 >= free1
    Y_ref = woq.qgemm(X, w, path="bf16_tc")
    assert fro_rel(Y2.cpu().numpy(), Y_ref.cpu().numpy()) <= BF16_READING_TOL
    assert torch.equal(Y, Y2)
    assert woq.device_status() == _lib.WOQ_OK
