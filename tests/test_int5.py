"""GPU parity of the int5 block-32 format against the CPU oracle, through the C ABI.

int5 (codes -16..15, scale max|w|/15) is a layout of this library's own: the soniqo English
guide, "INT5 vs INT8", deploys the decoder at 5 bits but gives no format. The CUDA-core GEMV
family (qgemv, qgemv_swiglu, qgemv_residual, qgemv_argmax, qgemv_chain, qgemm's FP32 path)
takes it at the FP32 paths' tolerance; the tensor-core forms refuse it.
"""

import numpy as np
import pytest
import torch

import oracle
import weight_only_bit_qgemv_b200 as woq
from weight_only_bit_qgemv_b200 import _lib, workloads
from tests.gpu_util import (FP32_TOL, guarded_out, max_rel, packed_from_weight, packed_raw,
                            ref_rows, tail_intact)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("m", [1, 2, 3, 8, 33, 64])
def test_qgemv_all_m(m):
    n, k = 1000, 2048
    w, p, s = packed_from_weight(workloads.weight(n, k, seed=50 + m), 5)
    x = workloads.activations(m, k, seed=60 + m)
    buf, y = guarded_out(m, n)
    woq.qgemv(x.cuda(), w, out=y)
    assert tail_intact(buf, m, n)
    assert max_rel(y.cpu().numpy(), ref_rows(x.numpy(), p, s, 5)) <= FP32_TOL


@pytest.mark.parametrize("proj", range(7))
def test_decoder_block_shapes_m1(proj):
    name, n, k = workloads.DECODER_PROJ[proj]
    w, p, s = packed_from_weight(workloads.weight(n, k, seed=workloads.layer_seed(0, proj)), 5)
    x = workloads.activations(1, k, seed=workloads.X_SEED)
    y = woq.qgemv(x.cuda(), w).cpu().numpy()
    assert max_rel(y, ref_rows(x.numpy(), p, s, 5)) <= FP32_TOL, name


@pytest.mark.parametrize("m", [1, 5])
def test_every_code_including_minus_16(m):
    w, p, s = packed_raw(517, 1024, 5, seed=9 + m)
    q = oracle.unpack(p, 5, 1024)
    assert q.min() == -16 and q.max() == 15
    x = workloads.activations(m, 1024, seed=3)
    y = woq.qgemv(x.cuda(), w).cpu().numpy()
    assert max_rel(y, ref_rows(x.numpy(), p, s, 5)) <= FP32_TOL


def test_lm_head_full_size_sampled():
    n, k = workloads.LM_HEAD
    w, p, s = packed_from_weight(workloads.weight(n, k, seed=workloads.LM_HEAD_SEED), 5)
    x = workloads.activations(1, k, seed=workloads.X_SEED)
    y = woq.qgemv(x.cuda(), w).cpu().numpy()
    rows = np.concatenate([np.random.default_rng(2).choice(n, 2048, replace=False), [0, n - 1]])
    assert max_rel(y[:, rows], ref_rows(x.numpy(), p, s, 5, rows)) <= FP32_TOL


def test_identity_closed_form():
    """W = I: s = fp16(1/15) = 0x2C44, code 15, so y = (1 - 2^-12) x."""
    K = 1024
    w, _, s = packed_from_weight(torch.eye(K), 5)
    assert int(s[0, 0]) == 0x2C44
    x = workloads.activations(1, K, seed=5)
    y = woq.qgemv(x.cuda(), w).cpu()
    torch.testing.assert_close(y, x * (1 - 2.0 ** -12), rtol=2e-7, atol=0)


def test_fused_epilogues_and_chain():
    """SwiGLU (rows interleaved), residual add, greedy pick and a two-item chain on int5."""
    Wg = workloads.weight(512, 1024, seed=71)
    Wu = workloads.weight(512, 1024, seed=72)
    wgu, pgu, sgu = packed_from_weight(woq.interleave_rows(Wg, Wu), 5)
    wd, pd, sd = packed_from_weight(workloads.weight(1024, 512, seed=73), 5)
    x = workloads.activations(2, 1024, seed=74)
    r = workloads.activations(2, 1024, seed=75)
    a = woq.qgemv_swiglu(x.cuda(), wgu)
    assert max_rel(a.cpu().numpy(), oracle.swiglu_ref(x.numpy(), pgu, sgu, 5)) <= FP32_TOL
    h = woq.qgemv_residual(a, wd, r.cuda())
    ref = oracle.residual_ref(a.cpu().numpy().astype(np.float64), pd, sd, 5, r.numpy())
    assert max_rel(h.cpu().numpy(), ref) <= FP32_TOL
    idx, val = woq.qgemv_argmax(x.cuda(), wgu)
    y = woq.qgemv(x.cuda(), wgu, path="cuda_core")
    assert torch.equal(idx.cpu(), torch.argmax(y, dim=1).cpu())
    a2 = torch.empty(2, 512, device="cuda")
    h2 = torch.empty(2, 1024, device="cuda")
    woq.qgemv_chain([woq.ChainItem(wgu, x.cuda(), a2, None, "swiglu"),
                     woq.ChainItem(wd, a2, h2, r.cuda(), "residual")], woq.chain_workspace())
    torch.cuda.synchronize()
    assert max_rel(a2.cpu().numpy(), oracle.swiglu_ref(x.numpy(), pgu, sgu, 5)) <= FP32_TOL
    ref2 = oracle.residual_ref(a2.cpu().numpy().astype(np.float64), pd, sd, 5, r.numpy())
    assert max_rel(h2.cpu().numpy(), ref2) <= FP32_TOL


def test_qgemm_fp32_path_and_refused_tensor_core_forms():
    n, k = 300, 1024
    w, p, s = packed_from_weight(workloads.weight(n, k, seed=81), 5)
    X = workloads.activations(100, k, seed=82)
    Y = woq.qgemm(X.cuda(), w)  # auto: the FP32 path for int5
    assert max_rel(Y.cpu().numpy(), ref_rows(X.numpy(), p, s, 5)) <= FP32_TOL
    assert woq.qgemm_workspace_bytes(100, w, "auto") == 0
    for path in ("bf16_tc", "split_tc"):
        with pytest.raises(woq.WoqError):
            woq.qgemm(X.cuda(), w, path=path)
    for path in ("split_tc", "split_gemm", "int8_tc"):
        with pytest.raises(woq.WoqError):
            woq.qgemv(X[:8].cuda(), w, path=path)
    assert woq.device_status() == _lib.WOQ_OK
