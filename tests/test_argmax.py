"""GPU tests of qgemv_argmax (fused greedy pick over a GEMV's outputs) against the oracle."""

import numpy as np
import pytest
import torch

import oracle
import weight_only_bit_qgemv_b200 as woq
from weight_only_bit_qgemv_b200 import workloads
from tests.gpu_util import FP32_TOL, packed_from_weight, packed_raw

pytestmark = pytest.mark.gpu


def _check(x, w, p, s, bits):
    """idx/val equal the greedy pick over the same kernel family's written outputs (same
    arithmetic), and the pick is valid against the exact float64 outputs."""
    xd = x.cuda()
    idx, val = woq.qgemv_argmax(xd, w)
    y = woq.qgemv(xd, w, path="cuda_core")
    torch.cuda.synchronize()
    gv, gi = torch.max(y, dim=1)  # first index of the maximum
    assert torch.equal(idx.cpu(), gi.cpu())
    assert torch.equal(val.cpu(), gv.cpu())
    ref = oracle.qgemv_ref(x.numpy(), p, s, bits)
    scale = np.abs(ref).max(axis=1)
    got = idx.cpu().numpy()
    rows = np.arange(ref.shape[0])
    assert np.all(ref[rows, got] >= ref.max(axis=1) - FP32_TOL * scale)
    assert np.all(np.abs(val.cpu().numpy() - ref[rows, got]) <= FP32_TOL * scale)


@pytest.mark.parametrize("m", [1, 2, 3, 8])
def test_lm_head_int8(m):
    n, k = workloads.LM_HEAD
    W = workloads.weight(n, k, seed=workloads.LM_HEAD_SEED)
    w, p, s = packed_from_weight(W, 8)
    _check(workloads.activations(m, k, seed=workloads.X_SEED + m), w, p, s, 8)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("n,k", [(3072, 1024), (1000, 2048), (40, 96)])
def test_shapes(bits, n, k):
    w, p, s = packed_raw(n, k, bits, seed=n + k)
    for m in (1, 4):
        _check(workloads.activations(m, k, seed=m), w, p, s, bits)


def test_ties_go_to_the_smallest_index():
    # rows 3, 700 and 1999 hold the same (largest) codes and scales: equal outputs
    n, k = 2048, 1024
    rng = np.random.default_rng(11)
    q = rng.integers(-3, 4, size=(n, k)).astype(np.int64)
    q[[3, 700, 1999]] = 7
    sb = np.full((n, k // 32), 0x3C00, dtype=np.uint16)  # every scale 1.0
    p = oracle.pack(q, 4)
    w = woq.PackedWeight(torch.from_numpy(p).cuda(), torch.from_numpy(sb.view(np.int16)).cuda(), 4, n, k)
    x = torch.ones(2, k)
    idx, val = woq.qgemv_argmax(x.cuda(), w)
    assert idx.cpu().tolist() == [3, 3]
    assert val.cpu().tolist() == [7.0 * k, 7.0 * k]


def test_nan_counts_as_the_maximum():
    w, _, _ = packed_raw(512, 256, 4, seed=3)
    x = torch.full((1, 256), float("nan"))
    idx, val = woq.qgemv_argmax(x.cuda(), w)
    assert idx.cpu().tolist() == [0] and torch.isnan(val.cpu()).all()


def test_deterministic_and_launch_count():
    n, k = workloads.LM_HEAD
    w, _, _ = packed_raw(n, k, 8, seed=5)
    x = workloads.activations(1, k, seed=9).cuda()
    before = woq.launch_count()
    a = woq.qgemv_argmax(x, w)
    b = woq.qgemv_argmax(x, w)
    torch.cuda.synchronize()
    assert woq.launch_count() - before == 6  # zero keys, GEMV, finish; twice
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
