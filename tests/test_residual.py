"""GPU parity of qgemv_residual (a decode projection with the residual add fused) against the
oracle, and of the wider-k reach of the fused-epilogue GEMVs."""

import pytest
import torch

import oracle
import weight_only_bit_qgemv_b200 as woq
from weight_only_bit_qgemv_b200 import workloads
from tests.gpu_util import FP32_TOL, guarded_out, max_rel, packed_from_weight, packed_raw, tail_intact

pytestmark = pytest.mark.gpu


def _stream(m, n, seed):
    """A residual stream with the magnitude of a decoder's hidden state."""
    g = torch.Generator().manual_seed(seed)
    return torch.randn(m, n, generator=g, dtype=torch.float32) * 4.0


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("proj", [3, 6])  # o [1024x2048], down [1024x3072]
@pytest.mark.parametrize("m", [1, 2, 5, 8, 64])
def test_decoder_o_and_down(bits, proj, m):
    name, n, k = workloads.DECODER_PROJ[proj]
    W = workloads.weight(n, k, seed=workloads.layer_seed(5, proj))
    w, p, s = packed_from_weight(W, bits)
    x = workloads.activations(m, k, seed=m + proj)
    r = _stream(m, n, seed=m)
    buf, y = guarded_out(m, n)
    woq.qgemv_residual(x.cuda(), w, r.cuda(), out=y)
    assert tail_intact(buf, m, n)
    ref = oracle.residual_ref(x.numpy(), p, s, bits, r.numpy())
    assert max_rel(y.cpu().numpy(), ref) <= FP32_TOL, name


@pytest.mark.parametrize("bits", [4, 8])
def test_in_place_update_of_the_stream(bits):
    n, k = 1024, 2048
    W = workloads.weight(n, k, seed=21)
    w, p, s = packed_from_weight(W, bits)
    for m in (1, 17):
        x = workloads.activations(m, k, seed=m)
        r = _stream(m, n, seed=m + 1)
        h = r.cuda().clone()
        out = woq.qgemv_residual(x.cuda(), w, h, out=h)
        assert out.data_ptr() == h.data_ptr()
        ref = oracle.residual_ref(x.numpy(), p, s, bits, r.numpy())
        assert max_rel(h.cpu().numpy(), ref) <= FP32_TOL


def test_equals_qgemv_plus_the_stream_bitwise():
    """The fused add is one FP32 add after the projection qgemv computes."""
    n, k = 1024, 2048
    W = workloads.weight(n, k, seed=22)
    w, _, _ = packed_from_weight(W, 4)
    for m in (1, 4, 40):
        x = workloads.activations(m, k, seed=m).cuda()
        r = _stream(m, n, seed=m).cuda()
        y = woq.qgemv_residual(x, w, r)
        assert torch.equal(y, woq.qgemv(x, w, path="cuda_core") + r)


@pytest.mark.parametrize("n,k", [(37, 96), (500, 2048), (1, 32), (130, 4096)])
def test_ragged(n, k):
    w, p, s = packed_raw(n, k, 8, seed=n + k)
    for m in (1, 3, 9):
        x = workloads.activations(m, k, seed=m)
        r = _stream(m, n, seed=m)
        buf, y = guarded_out(m, n)
        woq.qgemv_residual(x.cuda(), w, r.cuda(), out=y)
        assert tail_intact(buf, m, n)
        ref = oracle.residual_ref(x.numpy(), p, s, 8, r.numpy())
        assert max_rel(y.cpu().numpy(), ref) <= FP32_TOL


def test_long_rows_take_fewer_x_rows_per_cta():
    """k = 8192, int4, m = 64: the x rows of a CTA are halved until a stage fits; argmax and
    the residual add run where one x row and one stage fit."""
    n, k = 256, 8192
    W = workloads.weight(n, k, seed=23)
    w, p, s = packed_from_weight(W, 4)
    x = workloads.activations(64, k, seed=24)
    r = _stream(64, n, seed=25)
    y = woq.qgemv_residual(x.cuda(), w, r.cuda()).cpu().numpy()
    assert max_rel(y, oracle.residual_ref(x.numpy(), p, s, 4, r.numpy())) <= FP32_TOL
    x8 = x[:8].contiguous().cuda()
    idx, val = woq.qgemv_argmax(x8, w)
    gv, gi = torch.max(woq.qgemv(x8, w, path="cuda_core"), dim=1)  # the same FP32 outputs
    assert torch.equal(idx, gi) and torch.equal(val, gv)


def test_swiglu_at_k_4096_every_m():
    """qgemv_swiglu at k = 4096 (int8): fits at every m by halving the x rows per CTA."""
    i, k = 96, 4096
    Wg = workloads.weight(i, k, seed=26)
    Wu = workloads.weight(i, k, seed=27)
    w, p, s = packed_from_weight(woq.interleave_rows(Wg, Wu), 8)
    for m in (1, 7, 64):
        x = workloads.activations(m, k, seed=m)
        y = woq.qgemv_swiglu(x.cuda(), w).cpu().numpy()
        assert max_rel(y, oracle.swiglu_ref(x.numpy(), p, s, 8)) <= FP32_TOL


def test_one_launch_per_call():
    W = workloads.weight(1024, 3072, seed=28)
    w, _, _ = packed_from_weight(W, 4)
    x = workloads.activations(8, 3072, seed=1).cuda()
    r = _stream(8, 1024, seed=2).cuda()
    before = woq.launch_count()
    woq.qgemv_residual(x, w, r)
    assert woq.launch_count() - before == 1
    assert woq.device_status() == 0
