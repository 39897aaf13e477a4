"""GPU parity of qgemv (FP32 decode path) against the CPU oracle, through the C ABI."""

import numpy as np
import pytest
import torch

import weight_only_bit_qgemv_b200 as woq
from weight_only_bit_qgemv_b200 import workloads
from tests.gpu_util import (FP32_TOL, guarded_out, max_rel, packed_from_weight, packed_raw,
                            ref_rows, tail_intact)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("m", [1, 2, 3, 4, 7, 8, 16, 33, 64])
def test_qgemv_all_m(bits, m):
    n, k = 1000, 2048  # ragged n (not a multiple of any row grouping), two chunks per lane
    W = workloads.weight(n, k, seed=11 + m)
    w, p, s = packed_from_weight(W, bits)
    x = workloads.activations(m, k, seed=100 + m)
    y = woq.qgemv(x.cuda(), w).cpu().numpy()
    assert max_rel(y, ref_rows(x.numpy(), p, s, bits)) <= FP32_TOL


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("proj", range(7))
def test_decoder_block_shapes_m1(bits, proj):
    name, n, k = workloads.DECODER_PROJ[proj]
    W = workloads.weight(n, k, seed=workloads.layer_seed(0, proj))
    w, p, s = packed_from_weight(W, bits)
    x = workloads.activations(1, k, seed=workloads.X_SEED)
    y = woq.qgemv(x.cuda(), w).cpu().numpy()
    assert max_rel(y, ref_rows(x.numpy(), p, s, bits)) <= FP32_TOL, name


@pytest.mark.parametrize("bits", [8, 4])
def test_lm_head_full_size_sampled(bits):
    n, k = workloads.LM_HEAD
    W = workloads.weight(n, k, seed=workloads.LM_HEAD_SEED)
    w, p, s = packed_from_weight(W, bits)
    x = workloads.activations(1, k, seed=workloads.X_SEED)
    buf, y = guarded_out(1, n)
    woq.qgemv(x.cuda(), w, out=y)
    yc = y.cpu().numpy()
    assert tail_intact(buf, 1, n)
    assert np.all(np.isfinite(yc))
    rows = np.random.default_rng(0).choice(n, 2048, replace=False)
    rows = np.concatenate([rows, [0, 1, n - 2, n - 1]])
    assert max_rel(yc[:, rows], ref_rows(x.numpy(), p, s, bits, rows)) <= FP32_TOL


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("m", [1, 5])
def test_every_code_including_the_negative_extreme(bits, m):
    n, k = 257, 1024
    w, p, s = packed_raw(n, k, bits, seed=bits * 10 + m)
    x = workloads.activations(m, k, seed=3)
    y = woq.qgemv(x.cuda(), w).cpu().numpy()
    assert max_rel(y, ref_rows(x.numpy(), p, s, bits)) <= FP32_TOL


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("kind", ["one_hot", "ones", "alternating"])
def test_adversarial_x(bits, kind):
    n, k = 512, 1024
    w, p, s = packed_raw(n, k, bits, seed=77)
    x = np.zeros((3, k), dtype=np.float32)
    if kind == "one_hot":
        x[0, 0] = 1.0
        x[1, k - 1] = -2.0
        x[2, 517] = 3.0
    elif kind == "ones":
        x[:] = 1.0
    else:
        x[:, 0::2] = 1.0
        x[:, 1::2] = -1.0
        x[1] *= 1e-3
        x[2] *= 1e3
    y = woq.qgemv(torch.from_numpy(x).cuda(), w).cpu().numpy()
    ref = ref_rows(x, p, s, bits)
    for r in range(3):  # per x row: each row's own scale
        assert max_rel(y[r:r + 1], ref[r:r + 1]) <= FP32_TOL
    if kind == "one_hot":  # a single product per output: exact
        np.testing.assert_array_equal(y, ref.astype(np.float32))


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("n,k", [(1, 32), (31, 96), (33, 64), (129, 160), (4099, 512)])
def test_small_and_ragged_shapes(bits, n, k):
    W = workloads.weight(n, k, seed=n + k)
    w, p, s = packed_from_weight(W, bits)
    for m in (1, 3, 9):
        x = workloads.activations(m, k, seed=m)
        buf, y = guarded_out(m, n)
        woq.qgemv(x.cuda(), w, out=y)
        assert tail_intact(buf, m, n)
        assert max_rel(y.cpu().numpy(), ref_rows(x.numpy(), p, s, bits)) <= FP32_TOL


def test_zero_weight_gives_exact_zero():
    W = torch.zeros(300, 1024)
    w, _, _ = packed_from_weight(W, 4)
    y = woq.qgemv(workloads.activations(2, 1024, 1).cuda(), w)
    assert torch.count_nonzero(y).item() == 0


def test_identity_closed_form():
    K = 1024
    w, _, _ = packed_from_weight(torch.eye(K), 4)
    x = workloads.activations(1, K, seed=5)
    y = woq.qgemv(x.cuda(), w).cpu()
    torch.testing.assert_close(y, x * (1 - 2.0 ** -12), rtol=2e-7, atol=0)


def test_deterministic_bits():
    W = workloads.weight(3072, 1024, seed=1)
    w, _, _ = packed_from_weight(W, 4)
    x = workloads.activations(4, 1024, seed=2).cuda()
    a = woq.qgemv(x, w)
    b = woq.qgemv(x, w)
    assert torch.equal(a, b)


def test_launches_are_counted_and_stream_ordered():
    W = workloads.weight(2048, 1024, seed=3)
    w, p, s = packed_from_weight(W, 8)
    x = workloads.activations(1, 1024, seed=4)
    st = torch.cuda.Stream()
    before = woq.launch_count()
    with torch.cuda.stream(st):
        y = woq.qgemv(x.cuda(), w)
    st.synchronize()
    assert woq.launch_count() - before == 1
    assert max_rel(y.cpu().numpy(), ref_rows(x.numpy(), p, s, 8)) <= FP32_TOL


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("m", [8, 64])
@pytest.mark.parametrize("proj", [0, 3, 6])
def test_small_batch_tensor_core_decoder_shapes(bits, m, proj):
    """The tensor-core form (hi/lo bf16 split of x) keeps the FP32 tolerance."""
    name, n, k = workloads.DECODER_PROJ[proj]
    W = workloads.weight(n, k, seed=workloads.layer_seed(4, proj))
    w, p, s = packed_from_weight(W, bits)
    x = workloads.activations(m, k, seed=m)
    buf, y = guarded_out(m, n)
    woq.qgemv(x.cuda(), w, out=y, path="split_tc")
    assert tail_intact(buf, m, n)
    assert max_rel(y.cpu().numpy(), ref_rows(x.numpy(), p, s, bits)) <= FP32_TOL, name


def test_small_batch_lm_head_sampled():
    n, k = workloads.LM_HEAD
    W = workloads.weight(n, k, seed=workloads.LM_HEAD_SEED)
    w, p, s = packed_from_weight(W, 8)
    x = workloads.activations(16, k, seed=workloads.X_SEED)
    y = woq.qgemv(x.cuda(), w).cpu().numpy()
    rows = np.concatenate([np.random.default_rng(3).choice(n, 1024, replace=False), [n - 1]])
    assert max_rel(y[:, rows], ref_rows(x.numpy(), p, s, 8, rows)) <= FP32_TOL


def test_small_batch_wide_dynamic_range():
    """x spanning many binades: the two-term split keeps ~16 bits of each value."""
    n, k = 512, 1024
    w, p, s = packed_raw(n, k, 4, seed=31)
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((6, k)) * np.exp(rng.uniform(-8, 8, (6, k)))).astype(np.float32)
    y = woq.qgemv(torch.from_numpy(x).cuda(), w, path="split_tc").cpu().numpy()
    ref = ref_rows(x, p, s, 4)
    for r in range(6):
        assert max_rel(y[r:r + 1], ref[r:r + 1]) <= FP32_TOL


@pytest.mark.parametrize("m", [2, 3, 5, 17, 33])
def test_small_batch_tensor_core_ragged_rows(m):
    """Row counts that are not a multiple of the MMA's 8-column tile, on a ragged N."""
    n, k = 1000, 2048
    w, p, s = packed_raw(n, k, 4, seed=40 + m)
    x = workloads.activations(m, k, seed=m)
    buf, y = guarded_out(m, n)
    woq.qgemv(x.cuda(), w, out=y, path="split_tc")
    assert tail_intact(buf, m, n)
    assert max_rel(y.cpu().numpy(), ref_rows(x.numpy(), p, s, 4)) <= FP32_TOL


@pytest.mark.parametrize("bits", [4, 5, 8])
@pytest.mark.parametrize("n,k", [(1024, 2048), (1024, 3072), (1001, 2048), (999, 3072), (5, 4096),
                                 (300, 8192)])
def test_split_k_inside_the_cta(bits, n, k):
    """m = 1 over rows of more than 32 blocks: for int5 the 16-warp launch splits each row's K
    across 2 or 4 warps and adds their partial sums in a fixed order (int4 and int8 run the
    same shapes unsplit); ragged last tiles are read from global memory, and a matrix of fewer
    rows than one split tile takes the unsplit form."""
    W = workloads.weight(n, k, seed=n + k + bits)
    w, p, s = packed_from_weight(W, bits)
    x = workloads.activations(1, k, seed=k)
    buf, y = guarded_out(1, n)
    woq.qgemv(x.cuda(), w, out=y)
    assert tail_intact(buf, 1, n)
    assert torch.equal(y, woq.qgemv(x.cuda(), w))
    assert max_rel(y.cpu().numpy(), ref_rows(x.numpy(), p, s, bits)) <= FP32_TOL


def test_split_tc_rejects_shapes_outside_its_limits():
    w, _, _ = packed_raw(256, 96, 8, seed=5)  # k % 256 != 0
    x = workloads.activations(4, 96, seed=1).cuda()
    with pytest.raises(woq.WoqError):
        woq.qgemv(x, w, path="split_tc")
    x1 = workloads.activations(1, 96, seed=1).cuda()
    with pytest.raises(woq.WoqError):
        woq.qgemv(x1, w, path="split_tc")  # m = 1


def test_auto_and_cuda_core_paths_agree_bitwise_on_decoder_shapes():
    name, n, k = workloads.DECODER_PROJ[0]
    W = workloads.weight(n, k, seed=workloads.layer_seed(0, 0))
    w, _, _ = packed_from_weight(W, 4)
    x = workloads.activations(8, k, seed=2).cuda()
    a = woq.qgemv(x, w)
    b = woq.qgemv(x, w, path="cuda_core")
    assert torch.equal(a, b), name


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("proj", [0, 3, 6])
@pytest.mark.parametrize("m", [1, 24, 64])
def test_split_gemm_path(bits, proj, m):
    """qgemv through the tcgen05 split GEMM (x and s*q as bf16 hi + lo): FP32 tolerance."""
    name, n, k = workloads.DECODER_PROJ[proj]
    W = workloads.weight(n, k, seed=workloads.layer_seed(6, proj))
    w, p, s = packed_from_weight(W, bits)
    x = workloads.activations(m, k, seed=m + 3)
    buf, y = guarded_out(m, n)
    woq.qgemv(x.cuda(), w, out=y, path="split_gemm")
    assert tail_intact(buf, m, n)
    assert max_rel(y.cpu().numpy(), ref_rows(x.numpy(), p, s, bits)) <= FP32_TOL, name


def test_auto_routes_batched_decode_to_the_split_gemm():
    name, n, k = workloads.DECODER_PROJ[6]
    W = workloads.weight(n, k, seed=7)
    w, _, _ = packed_from_weight(W, 4)
    for m, same_as in ((15, "cuda_core"), (16, "split_gemm"), (64, "split_gemm")):
        x = workloads.activations(m, k, seed=m).cuda()
        assert torch.equal(woq.qgemv(x, w), woq.qgemv(x, w, path=same_as)), (m, same_as)


@pytest.mark.parametrize("bits", [4, 8])
def test_auto_routes_on_a_wide_matrix(bits):
    """Rows enough for one 128-row tile per SM and more: the measured choice by m and width."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    n, k = 128 * sms + 1000, 512
    W = workloads.weight(n, k, seed=70 + bits)
    w, p, s = packed_from_weight(W, bits)
    mid = "int8_tc" if bits == 8 else "split_tc"
    for m, same_as in ((2, "cuda_core"), (3, mid), (4, mid), (5, "split_tc"), (32, "split_tc"),
                       (33, "split_gemm")):
        x = workloads.activations(m, k, seed=m)
        a = woq.qgemv(x.cuda(), w)
        assert torch.equal(a, woq.qgemv(x.cuda(), w, path=same_as)), (m, same_as)
        rows = np.concatenate([np.random.default_rng(m).choice(n, 256, replace=False), [n - 1]])
        assert max_rel(a.cpu().numpy()[:, rows], ref_rows(x.numpy(), p, s, bits, rows)) <= FP32_TOL
