"""GPU parity of qgemm (tcgen05 bf16 prefill path and the FP32 path) against the oracle."""

import numpy as np
import pytest
import torch

import oracle
import weight_only_bit_qgemv_b200 as woq
from weight_only_bit_qgemv_b200 import workloads
from tests.gpu_util import (BF16_READING_TOL, BF16_TOL, FP32_TOL, fro_rel, guarded_out, max_rel,
                            packed_from_weight, packed_raw, ref_rows, tail_intact)

pytestmark = pytest.mark.gpu


def _check_bf16(y, X, p, s, bits, rows=None):
    if rows is not None:
        p, s, y = p[rows], s[rows], y[:, rows]
    exact = oracle.qgemv_ref(X, p, s, bits)
    reading = oracle.qgemm_bf16_ref(X, p, s, bits)
    assert fro_rel(y, exact) <= BF16_TOL
    assert fro_rel(y, reading) <= BF16_READING_TOL


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("m", [1, 65, 128, 137, 375, 512])
def test_bf16_tc_decoder_q_shape(bits, m):
    n, k = 2048, 1024
    W = workloads.weight(n, k, seed=workloads.layer_seed(1, 0))
    w, p, s = packed_from_weight(W, bits)
    X = workloads.activations(m, k, seed=workloads.X_SEED)
    buf, Y = guarded_out(m, n)
    woq.qgemm(X.cuda(), w, path="bf16_tc", out=Y)
    assert tail_intact(buf, m, n)
    _check_bf16(Y.cpu().numpy(), X.numpy(), p, s, bits)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("proj", range(7))
def test_bf16_tc_every_decoder_shape_m512(bits, proj):
    name, n, k = workloads.DECODER_PROJ[proj]
    W = workloads.weight(n, k, seed=workloads.layer_seed(2, proj))
    w, p, s = packed_from_weight(W, bits)
    X = workloads.activations(512, k, seed=workloads.X_SEED)
    Y = woq.qgemm(X.cuda(), w, path="bf16_tc").cpu().numpy()
    _check_bf16(Y, X.numpy(), p, s, bits)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("n,k", [(130, 96), (1000, 160), (256, 32), (8, 3072)])
def test_bf16_tc_ragged(bits, n, k):
    W = workloads.weight(n, k, seed=n * 3 + k)
    w, p, s = packed_from_weight(W, bits)
    for m in (200, 129):
        X = workloads.activations(m, k, seed=m)
        buf, Y = guarded_out(m, n)
        woq.qgemm(X.cuda(), w, path="bf16_tc", out=Y)
        assert tail_intact(buf, m, n)
        _check_bf16(Y.cpu().numpy(), X.numpy(), p, s, bits)


@pytest.mark.parametrize("bits", [4, 8])
def test_bf16_tc_every_code(bits):
    w, p, s = packed_raw(384, 1024, bits, seed=5)
    X = workloads.activations(256, 1024, seed=6)
    Y = woq.qgemm(X.cuda(), w, path="bf16_tc").cpu().numpy()
    _check_bf16(Y, X.numpy(), p, s, bits)


def test_bf16_tc_long_prefill_sampled():
    """M = 4096 at a decoder shape, full launch; oracle on sampled rows and columns."""
    n, k = 3072, 1024
    W = workloads.weight(n, k, seed=workloads.layer_seed(3, 4))
    w, p, s = packed_from_weight(W, 4)
    X = workloads.activations(4096, k, seed=workloads.X_SEED)
    Y = woq.qgemm(X.cuda(), w, path="bf16_tc").cpu().numpy()
    rng = np.random.default_rng(1)
    mr = np.concatenate([rng.choice(4096, 96, replace=False), [0, 4095]])
    nr = np.concatenate([rng.choice(n, 512, replace=False), [0, n - 1]])
    _check_bf16(Y[mr], X.numpy()[mr], p, s, 4, rows=nr)


def test_bf16_tc_lm_head_int8_sampled():
    n, k = workloads.LM_HEAD
    W = workloads.weight(n, k, seed=workloads.LM_HEAD_SEED)
    w, p, s = packed_from_weight(W, 8)
    X = workloads.activations(128, k, seed=workloads.X_SEED)
    buf, Y = guarded_out(128, n)
    woq.qgemm(X.cuda(), w, path="bf16_tc", out=Y)
    assert tail_intact(buf, 128, n)
    nr = np.concatenate([np.random.default_rng(2).choice(n, 1024, replace=False), [n - 1]])
    _check_bf16(Y.cpu().numpy(), X.numpy(), p, s, 8, rows=nr)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("m", [1, 65, 200])
def test_fp32_path_any_m(bits, m):
    n, k = 1024, 1024
    W = workloads.weight(n, k, seed=m)
    w, p, s = packed_from_weight(W, bits)
    X = workloads.activations(m, k, seed=m + 1)
    assert woq.qgemm_workspace_bytes(m, w, "fp32") == 0
    Y = woq.qgemm(X.cuda(), w, path="fp32").cpu().numpy()
    assert max_rel(Y, ref_rows(X.numpy(), p, s, bits)) <= FP32_TOL


def test_auto_path_picks_by_m():
    W = workloads.weight(256, 1024, seed=9)
    w, p, s = packed_from_weight(W, 4)
    # below 128 rows: the CUDA-core kernel or the split tensor-core form, no workspace
    assert woq.qgemm_workspace_bytes(23, w, "auto") == 0
    assert woq.qgemm_workspace_bytes(64, w, "auto") == 0
    # from 128 rows: the bf16 copy of X, plus FP32 partials when the plan splits K
    assert woq.qgemm_workspace_bytes(128, w, "auto") == woq.qgemm_workspace_bytes(128, w, "bf16_tc")
    for m in (8, 64):  # both FP32-accurate paths
        X = workloads.activations(m, 1024, seed=1)
        Y = woq.qgemm(X.cuda(), w).cpu().numpy()
        assert max_rel(Y, ref_rows(X.numpy(), p, s, 4)) <= FP32_TOL


@pytest.mark.parametrize("m,n,k", [(512, 1024, 3072), (128, 2048, 1024), (64, 4096, 1024)])
def test_bf16_tc_split_k_shapes(m, n, k):
    """Shapes whose plan splits K across CTAs (few output tiles); partials summed in order."""
    W = workloads.weight(n, k, seed=m + n)
    w, p, s = packed_from_weight(W, 4)
    X = workloads.activations(m, k, seed=k)
    buf, Y = guarded_out(m, n)
    ws = torch.empty(woq.qgemm_workspace_bytes(m, w, "bf16_tc"), dtype=torch.uint8, device="cuda")
    woq.qgemm(X.cuda(), w, path="bf16_tc", out=Y, workspace=ws)
    assert tail_intact(buf, m, n)
    _check_bf16(Y.cpu().numpy(), X.numpy(), p, s, 4)
    Y2 = woq.qgemm(X.cuda(), w, path="bf16_tc", workspace=ws)
    assert torch.equal(Y, Y2)


def test_bf16_tc_deterministic_and_counted():
    W = workloads.weight(1024, 2048, seed=4)
    w, _, _ = packed_from_weight(W, 4)
    X = workloads.activations(300, 2048, seed=5).cuda()
    before = woq.launch_count()
    a = woq.qgemm(X, w, path="bf16_tc")
    b = woq.qgemm(X, w, path="bf16_tc")
    assert torch.equal(a, b)
    # conversion + GEMM (+ split-K reduction when the plan splits K), twice
    assert woq.launch_count() - before in (4, 6)
    assert woq.device_status() == 0
