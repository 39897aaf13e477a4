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


def test_split_tc_workspace_and_determinism():
    """Workspace covers 128 bf16 rows (hi + lo) per 64-row tile; repeated calls agree bitwise;
    each call launches the X split, the GEMM and, when K is split, the reduction."""
    n, k = 1024, 3072
    W = workloads.weight(n, k, seed=12)
    w, p, s = packed_from_weight(W, 4)
    for m in (1, 64, 65):
        assert woq.qgemm_workspace_bytes(m, w, "split_tc") >= ((m + 63) // 64) * 128 * k * 2
    X = workloads.activations(64, k, seed=13).cuda()
    ws = torch.empty(woq.qgemm_workspace_bytes(64, w, "split_tc"), dtype=torch.uint8, device="cuda")
    before = woq.launch_count()
    a = woq.qgemm(X, w, path="split_tc", workspace=ws)
    b = woq.qgemm(X, w, path="split_tc", workspace=ws)
    assert torch.equal(a, b)
    assert woq.launch_count() - before in (4, 6)
    assert woq.device_status() == 0
    assert max_rel(a.cpu().numpy(), ref_rows(X.cpu().numpy(), p, s, 4)) <= FP32_TOL


def test_split_tc_too_small_workspace_is_refused():
    W = workloads.weight(256, 1024, seed=14)
    w, _, _ = packed_from_weight(W, 4)
    X = workloads.activations(16, 1024, seed=15).cuda()
    need = woq.qgemm_workspace_bytes(16, w, "split_tc")
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(woq.WoqError):
        woq.qgemm(X, w, path="split_tc", workspace=ws)
