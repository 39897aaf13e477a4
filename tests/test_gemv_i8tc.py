"""GPU parity of qgemv's integer tensor-core form (WOQ_GEMV_INT8_TC) against the CPU oracle.

The form writes each 32-block of x as 2^E (d0 + d1 2^-7 + d2 2^-14) with small integer digits,
multiplies the codes by the digits exactly on the tensor cores, and scales and accumulates the
block sums in FP32; it is held to the FP32 paths' tolerance.
"""

import numpy as np
import pytest
import torch

import weight_only_bit_qgemv_b200 as woq
from weight_only_bit_qgemv_b200 import workloads
from tests.gpu_util import (FP32_TOL, guarded_out, max_rel, packed_from_weight, packed_raw,
                            ref_rows, tail_intact)

pytestmark = pytest.mark.gpu


def run(x_np, w, m, n):
    buf, y = guarded_out(m, n)
    woq.qgemv(torch.from_numpy(np.ascontiguousarray(x_np)).cuda(), w, out=y, path="int8_tc")
    assert tail_intact(buf, m, n)
    return y.cpu().numpy()


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("m", [1, 2, 3, 4])
@pytest.mark.parametrize("proj", range(7))
def test_decoder_shapes(bits, m, proj):
    """Every decoder projection (K split across clusters of 3 to 8 CTAs)."""
    name, n, k = workloads.DECODER_PROJ[proj]
    W = workloads.weight(n, k, seed=workloads.layer_seed(2, proj))
    w, p, s = packed_from_weight(W, bits)
    x = workloads.activations(m, k, seed=50 + m)
    y = run(x.numpy(), w, m, n)
    assert max_rel(y, ref_rows(x.numpy(), p, s, bits)) <= FP32_TOL, name


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("n,k", [(1000, 2048), (4099, 512), (33, 128), (128, 3072), (300, 4096)])
def test_ragged_rows_and_k(bits, n, k):
    W = workloads.weight(n, k, seed=n + k)
    w, p, s = packed_from_weight(W, bits)
    for m in (1, 3):
        x = workloads.activations(m, k, seed=m + 9)
        y = run(x.numpy(), w, m, n)
        assert max_rel(y, ref_rows(x.numpy(), p, s, bits)) <= FP32_TOL


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("m", [1, 4])
def test_every_code_including_the_negative_extreme(bits, m):
    w, p, s = packed_raw(1000, 1024, bits, seed=bits + m)
    x = workloads.activations(m, 1024, seed=4)
    y = run(x.numpy(), w, m, 1000)
    assert max_rel(y, ref_rows(x.numpy(), p, s, bits)) <= FP32_TOL


@pytest.mark.parametrize("bits", [4, 8])
def test_wide_dynamic_range_and_extreme_magnitudes(bits):
    """x spanning e^-8..e^8 inside blocks, rows of 1e-30 and 1e30 scale, and zero blocks:
    each activation row keeps the tolerance on its own scale."""
    n, k = 512, 1024
    w, p, s = packed_raw(n, k, bits, seed=31)
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((4, k)) * np.exp(rng.uniform(-8, 8, (4, k)))).astype(np.float32)
    x[1] *= np.float32(1e-30)
    x[2] *= np.float32(1e30)
    x[3, 64:256] = 0.0
    y = run(x, w, 4, n)
    ref = ref_rows(x, p, s, bits)
    for r in range(4):
        assert max_rel(y[r:r + 1], ref[r:r + 1]) <= FP32_TOL, r


@pytest.mark.parametrize("bits", [4, 8])
def test_one_hot_is_exact_and_zero_gives_zero(bits):
    n, k = 256, 512
    w, p, s = packed_raw(n, k, bits, seed=8)
    x = np.zeros((3, k), dtype=np.float32)
    x[0, 0] = 1.0
    x[1, k - 1] = -2.5
    y = run(x, w, 3, n)
    ref = ref_rows(x, p, s, bits)
    np.testing.assert_array_equal(y, ref.astype(np.float32))
    assert np.count_nonzero(y[2]) == 0


def test_nan_in_a_block_makes_its_outputs_nan():
    n, k = 256, 1024
    w, _, _ = packed_raw(n, k, 4, seed=9)
    x = workloads.activations(2, k, seed=3).numpy()
    x[1, 77] = np.nan
    y = run(x, w, 2, n)
    assert np.all(np.isfinite(y[0])) and np.all(np.isnan(y[1]))


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("m", [1, 2])
def test_lm_head_full_size_sampled(bits, m):
    """The 151936-row lm_head: persistent CTAs walking 128-row tiles over the whole of K."""
    n, k = workloads.LM_HEAD
    W = workloads.weight(n, k, seed=workloads.LM_HEAD_SEED)
    w, p, s = packed_from_weight(W, bits)
    x = workloads.activations(m, k, seed=workloads.X_SEED)
    y = run(x.numpy(), w, m, n)
    assert np.all(np.isfinite(y))
    rows = np.concatenate([np.random.default_rng(1).choice(n, 2048, replace=False), [0, 127, 128, n - 1]])
    assert max_rel(y[:, rows], ref_rows(x.numpy(), p, s, bits, rows)) <= FP32_TOL


def test_deterministic_and_stream_ordered():
    W = workloads.weight(3072, 1024, seed=1)
    w, _, _ = packed_from_weight(W, 4)
    x = workloads.activations(2, 1024, seed=2).cuda()
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        a = woq.qgemv(x, w, path="int8_tc")
        b = woq.qgemv(x, w, path="int8_tc")
    st.synchronize()
    assert torch.equal(a, b)
    assert woq.device_status() == 0


def test_captured_in_a_cuda_graph():
    W = workloads.weight(1024, 3072, seed=5)
    w, p, s = packed_from_weight(W, 4)
    x = workloads.activations(1, 3072, seed=6)
    xd = x.cuda()
    y = torch.empty(1, 1024, device="cuda")
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        woq.qgemv(xd, w, out=y, path="int8_tc", stream=st)
    st.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        woq.qgemv(xd, w, out=y, path="int8_tc", stream=st)
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert max_rel(y.cpu().numpy(), ref_rows(x.numpy(), p, s, 4)) <= FP32_TOL


def test_rejects_shapes_outside_its_limits():
    w, _, _ = packed_raw(256, 96, 8, seed=5)  # k % 128 != 0
    with pytest.raises(woq.WoqError):
        woq.qgemv(workloads.activations(1, 96, seed=1).cuda(), w, path="int8_tc")
    w2, _, _ = packed_raw(256, 256, 8, seed=5)
    with pytest.raises(woq.WoqError):
        woq.qgemv(workloads.activations(5, 256, seed=1).cuda(), w2, path="int8_tc")  # m > 4
