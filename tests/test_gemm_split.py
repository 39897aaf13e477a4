"""GPU parity of qgemm's FP32-accurate tensor-core path (split_tc) against the oracle.

Both operands go to the tcgen05 tensor cores as bf16 hi + bf16 lo pairs (64 activation rows
per tile), so the result must meet the FP32 tolerance, not the bf16 one.
"""

import numpy as np
import pytest
import torch

import weight_only_bit_qgemv_b200 as woq
from weight_only_bit_qgemv_b200 import workloads
from tests.gpu_util import (FP32_TOL, guarded_out, max_rel, packed_from_weight, packed_raw,
                            ref_rows, tail_intact)

pytestmark = pytest.mark.gpu


def _run(X: torch.Tensor, w, m: int, n: int):
    buf, Y = guarded_out(m, n)
    woq.qgemm(X.cuda(), w, path="split_tc", out=Y)
    assert tail_intact(buf, m, n)
    return Y.cpu().numpy()


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("proj", range(7))
@pytest.mark.parametrize("m", [1, 16, 64])
def test_split_tc_every_decoder_shape(bits, proj, m):
    name, n, k = workloads.DECODER_PROJ[proj]
    W = workloads.weight(n, k, seed=workloads.layer_seed(4, proj))
    w, p, s = packed_from_weight(W, bits)
    X = workloads.activations(m, k, seed=workloads.X_SEED + m)
    Y = _run(X, w, m, n)
    assert max_rel(Y, ref_rows(X.numpy(), p, s, bits)) <= FP32_TOL, name


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("m", [2, 33, 65, 130, 300])
def test_split_tc_ragged_rows_several_tiles(bits, m):
    """Row counts spanning several 64-row tiles with a ragged last one."""
    n, k = 1000, 2048
    w, p, s = packed_raw(n, k, bits, seed=50 + m)
    X = workloads.activations(m, k, seed=m)
    Y = _run(X, w, m, n)
    assert max_rel(Y, ref_rows(X.numpy(), p, s, bits)) <= FP32_TOL


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("n,k", [(130, 96), (1000, 160), (256, 32), (8, 3072), (64, 8192)])
def test_split_tc_ragged_shapes(bits, n, k):
    W = workloads.weight(n, k, seed=n * 5 + k)
    w, p, s = packed_from_weight(W, bits)
    for m in (7, 64):
        X = workloads.activations(m, k, seed=m + k)
        Y = _run(X, w, m, n)
        assert max_rel(Y, ref_rows(X.numpy(), p, s, bits)) <= FP32_TOL


@pytest.mark.parametrize("bits", [4, 8])
def test_split_tc_every_code(bits):
    """Uniform codes (the extreme ones included) and random scales."""
    w, p, s = packed_raw(384, 1024, bits, seed=8)
    X = workloads.activations(40, 1024, seed=9)
    Y = _run(X, w, 40, 384)
    assert max_rel(Y, ref_rows(X.numpy(), p, s, bits)) <= FP32_TOL


def test_split_tc_wide_dynamic_range():
    """x spanning e^-8 .. e^8: the two-term split keeps about 16 bits of every value."""
    n, k = 512, 1024
    w, p, s = packed_raw(n, k, 4, seed=33)
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((24, k)) * np.exp(rng.uniform(-8, 8, (24, k)))).astype(np.float32)
    Y = _run(torch.from_numpy(x), w, 24, n)
    ref = ref_rows(x, p, s, 4)
    for r in range(24):
        assert max_rel(Y[r:r + 1], ref[r:r + 1]) <= FP32_TOL


def test_split_tc_lm_head_int8_sampled():
    n, k = workloads.LM_HEAD
    W = workloads.weight(n, k, seed=workloads.LM_HEAD_SEED)
    w, p, s = packed_from_weight(W, 8)
    X = workloads.activations(64, k, seed=workloads.X_SEED)
    Y = _run(X, w, 64, n)
    rows = np.concatenate([np.random.default_rng(6).choice(n, 1024, replace=False), [0, n - 1]])
    assert max_rel(Y[:, rows], ref_rows(X.numpy(), p, s, 8, rows)) <= FP32_TOL


def test_split_tc_one_launch_no_workspace_deterministic():
    """No workspace; one launch per call (K-splits summed inside their cluster); repeated calls
    agree bitwise, with and without K-splits."""
    for n, k in ((1024, 3072), (6144, 1024), (4096, 1024)):
        W = workloads.weight(n, k, seed=12 + n)
        w, p, s = packed_from_weight(W, 4)
        for m in (1, 64, 65):
            assert woq.qgemm_workspace_bytes(m, w, "split_tc") == 0
        X = workloads.activations(64, k, seed=13).cuda()
        before = woq.launch_count()
        a = woq.qgemm(X, w, path="split_tc")
        b = woq.qgemm(X, w, path="split_tc")
        assert woq.launch_count() - before == 2
        assert torch.equal(a, b)
        assert woq.device_status() == 0
        assert max_rel(a.cpu().numpy(), ref_rows(X.cpu().numpy(), p, s, 4)) <= FP32_TOL


def test_split_tc_in_a_cuda_graph():
    """Captured and replayed: the cluster launch and its on-chip reduction replay correctly."""
    n, k = 1024, 2048
    W = workloads.weight(n, k, seed=16)
    w, p, s = packed_from_weight(W, 8)
    X = workloads.activations(48, k, seed=17).cuda()
    Y = torch.empty(48, n, device="cuda")
    woq.qgemm(X, w, path="split_tc", out=Y)  # warm-up outside the capture
    g = torch.cuda.CUDAGraph()
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        with torch.cuda.graph(g, stream=st):
            woq.qgemm(X, w, path="split_tc", out=Y, stream=st)
    Y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert max_rel(Y.cpu().numpy(), ref_rows(X.cpu().numpy(), p, s, 8)) <= FP32_TOL
