"""GPU parity of qgemv_swiglu (gate|up GEMV with a fused SwiGLU) against the oracle."""

import pytest
import torch

import oracle
import weight_only_bit_qgemv_b200 as woq
from weight_only_bit_qgemv_b200 import workloads
from tests.gpu_util import FP32_TOL, max_rel, packed_from_weight

pytestmark = pytest.mark.gpu


def _gate_up(i, k, seed):
    Wg = workloads.weight(i, k, seed=seed)
    Wu = workloads.weight(i, k, seed=seed + 1)
    return woq.interleave_rows(Wg, Wu)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("m", [1, 2, 5, 8, 64])
def test_decoder_gate_up(bits, m):
    W = _gate_up(3072, 1024, seed=workloads.layer_seed(3, 4))
    w, p, s = packed_from_weight(W, bits)
    x = workloads.activations(m, 1024, seed=m)
    y = woq.qgemv_swiglu(x.cuda(), w).cpu().numpy()
    ref = oracle.swiglu_ref(x.numpy(), p, s, bits)
    assert y.shape == (m, 3072)
    assert max_rel(y, ref) <= FP32_TOL


@pytest.mark.parametrize("i,k", [(37, 96), (500, 2048), (1, 32)])
def test_ragged(i, k):
    W = _gate_up(i, k, seed=i + k)
    w, p, s = packed_from_weight(W, 4)
    for m in (1, 3):
        x = workloads.activations(m, k, seed=m)
        out = torch.full((m, i + 8), 7.0, device="cuda")
        y = out[:, :i].contiguous()
        woq.qgemv_swiglu(x.cuda(), w, out=y)
        assert max_rel(y.cpu().numpy(), oracle.swiglu_ref(x.numpy(), p, s, 4)) <= FP32_TOL


def test_gate_and_up_match_the_plain_gemv_outputs():
    """silu(g) * u from the fused kernel equals the same product over qgemv's written outputs
    up to the SiLU's own rounding."""
    W = _gate_up(1024, 1024, seed=5)
    w, _, _ = packed_from_weight(W, 4)
    x = workloads.activations(2, 1024, seed=4).cuda()
    y = woq.qgemv_swiglu(x, w)
    full = woq.qgemv(x, w, path="cuda_core")
    g, u = full[:, 0::2].double(), full[:, 1::2].double()
    expect = (g * torch.sigmoid(g) * u).float()
    assert torch.allclose(y, expect, rtol=2e-6, atol=1e-6 * expect.abs().max().item())


def test_odd_n_is_rejected():
    w, _, _ = packed_from_weight(workloads.weight(3, 64, seed=1), 4)
    with pytest.raises(woq.WoqError):
        woq.qgemv_swiglu(workloads.activations(1, 64, seed=1).cuda(), w, out=torch.empty(1, 1, device="cuda"))
