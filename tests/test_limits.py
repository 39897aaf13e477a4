"""GPU parity at the documented maximum sizes of every entry point, and the first size past
each limit returning its status with nothing written.

The limits are those of include/woq.h: qgemv k <= 32768 (int5 10752) and m <= 64; qgemv_swiglu and
qgemv_residual k <= 8192 while a stage of weight rows and a CTA's x rows fit in shared
memory (int4 SwiGLU up to 7168, int8 residual up to 7680); qgemv_argmax m <= 8 and the same
k rule; qgemv_chain m <= 8, k <= 8192 (at m = 8 about 5600, where its staged x rows still
leave room for two weight stages) and at most 8 items.
"""

import numpy as np
import pytest
import torch

import oracle
import weight_only_bit_qgemv_b200 as woq
from weight_only_bit_qgemv_b200 import workloads
from tests.gpu_util import FP32_TOL, guarded_out, max_rel, packed_from_weight, ref_rows, tail_intact

pytestmark = pytest.mark.gpu


def _np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


@pytest.mark.parametrize("bits,k", [(4, 32768), (8, 32768), (5, 10752)])
@pytest.mark.parametrize("m", [1, 2, 5, 64])
def test_qgemv_at_the_largest_k(bits, k, m):
    """k = 32768: x rows no longer fit the staged kernel's budget, so the register-path kernel
    takes the call. int5 runs on the staged kernel only: one x row per CTA up to k = 10752."""
    n = 300
    W = workloads.weight(n, k, seed=bits + m)
    w, p, s = packed_from_weight(W, bits)
    x = workloads.activations(m, k, seed=m)
    buf, y = guarded_out(m, n)
    woq.qgemv(x.cuda(), w, out=y, path="cuda_core")
    assert tail_intact(buf, m, n)
    assert max_rel(_np(y), ref_rows(x.numpy(), p, s, bits)) <= FP32_TOL


def test_qgemv_past_the_largest_k_or_m_is_refused():
    # int5 with 2000 rows: the 4-way split form (4-row stages) is not taken, 8-row stages
    # do not fit beside the x row
    for bits, k, n in ((4, 32800, 64), (5, 10880, 2000)):
        w, _, _ = packed_from_weight(workloads.weight(n, k, seed=1), bits)
        with pytest.raises(woq.WoqError) as e:
            woq.qgemv(workloads.activations(1, k, seed=1).cuda(), w)
        assert e.value.status == -2, bits  # WOQ_ESHAPE
    w2, _, _ = packed_from_weight(workloads.weight(64, 256, seed=2), 4)
    y = torch.full((65, 64), 7.0, device="cuda")
    with pytest.raises(woq.WoqError) as e:
        woq.qgemv(workloads.activations(65, 256, seed=2).cuda(), w2, out=y)
    assert e.value.status == -1  # WOQ_EINVAL
    assert torch.all(y == 7.0)


@pytest.mark.parametrize("bits,k", [(4, 7168), (8, 4096)])
def test_swiglu_at_its_largest_k(bits, k):
    n = 2 * 96
    W = workloads.weight(n, k, seed=k)
    w, p, s = packed_from_weight(W, bits)
    x = workloads.activations(64, k, seed=3)
    a = woq.qgemv_swiglu(x.cuda(), w)
    assert max_rel(_np(a), oracle.swiglu_ref(x.numpy(), p, s, bits)) <= FP32_TOL


def test_swiglu_past_its_shared_memory_budget_is_refused():
    w, _, _ = packed_from_weight(workloads.weight(64, 8192, seed=4), 4)
    with pytest.raises(woq.WoqError) as e:
        woq.qgemv_swiglu(workloads.activations(1, 8192, seed=4).cuda(), w)
    assert e.value.status == -2


@pytest.mark.parametrize("bits,k", [(4, 8192), (5, 8192), (8, 7680)])
def test_residual_at_its_largest_k(bits, k):
    n = 200
    W = workloads.weight(n, k, seed=k + bits)
    w, p, s = packed_from_weight(W, bits)
    x = workloads.activations(64, k, seed=5)
    r = workloads.activations(64, n, seed=6)
    y = woq.qgemv_residual(x.cuda(), w, r.cuda())
    assert max_rel(_np(y), oracle.residual_ref(x.numpy(), p, s, bits, r.numpy())) <= FP32_TOL


def test_residual_past_its_shared_memory_budget_is_refused():
    w, _, _ = packed_from_weight(workloads.weight(64, 8192, seed=7), 8)
    with pytest.raises(woq.WoqError) as e:
        woq.qgemv_residual(workloads.activations(1, 8192, seed=7).cuda(), w,
                           workloads.activations(1, 64, seed=8).cuda())
    assert e.value.status == -2


@pytest.mark.parametrize("bits,k", [(4, 8192), (8, 7680)])
def test_argmax_at_its_largest_m_and_k(bits, k):
    n = 500
    W = workloads.weight(n, k, seed=k + 1)
    w, p, s = packed_from_weight(W, bits)
    x = workloads.activations(8, k, seed=9)
    idx, val = woq.qgemv_argmax(x.cuda(), w)
    ref = oracle.qgemv_ref(x.numpy(), p, s, bits)
    scale = np.abs(ref).max(axis=1)
    got = _np(idx)
    rows = np.arange(8)
    assert np.all(ref[rows, got] >= ref.max(axis=1) - FP32_TOL * scale)
    assert np.all(np.abs(_np(val) - ref[rows, got]) <= FP32_TOL * scale)


def test_argmax_past_its_largest_m_is_refused():
    w, _, _ = packed_from_weight(workloads.weight(64, 256, seed=10), 4)
    with pytest.raises(woq.WoqError) as e:
        woq.qgemv_argmax(workloads.activations(9, 256, seed=10).cuda(), w)
    assert e.value.status == -1


@pytest.mark.parametrize("m,k0", [(4, 8192), (8, 4096)])
def test_chain_with_the_most_items_at_the_largest_m_and_k(m, k0):
    """8 items (the most a chain takes) at the largest k that m allows (x rows of m = 8 at
    k = 8192 do not fit beside two weight stages): each item reads the previous item's
    output, with the plain, SwiGLU and residual epilogues."""
    ks = [k0, 512, 256, 512, 256, 256, 256, 512]
    ns = [512, 512, 512, 512, 256, 512, 512, 512]
    eps = ["none", "swiglu", "none", "swiglu", "residual", "swiglu", "none", "residual"]
    ws = []
    for i, (n, k) in enumerate(zip(ns, ks)):
        ws.append(packed_from_weight(workloads.weight(n, k, seed=20 + i), 4))
    x0 = workloads.activations(m, ks[0], seed=30)
    bufs, items = [], []
    prev = x0.cuda()
    prev_np = x0.numpy().astype(np.float64)
    refs = []
    for i, ((w, p, s), ep) in enumerate(zip(ws, eps)):
        n_out = ns[i] // 2 if ep == "swiglu" else ns[i]
        out = torch.empty(m, n_out, device="cuda")
        if ep == "residual":
            r = workloads.activations(m, n_out, seed=40 + i)
            rd = r.cuda()
            items.append(woq.ChainItem(w, prev, out, rd, ep))
            ref = oracle.residual_ref(prev_np, p, s, 4, r.numpy())
        elif ep == "swiglu":
            items.append(woq.ChainItem(w, prev, out, None, ep))
            ref = oracle.swiglu_ref(prev_np, p, s, 4)
        else:
            items.append(woq.ChainItem(w, prev, out, None, ep))
            ref = oracle.qgemv_ref(prev_np, p, s, 4)
        bufs.append(out)
        refs.append(ref)
        prev, prev_np = out, ref
        if i + 1 < len(ks):
            assert ks[i + 1] == n_out  # the next item's input width
    woq.qgemv_chain(items, woq.chain_workspace())
    torch.cuda.synchronize()
    for i, (b, ref) in enumerate(zip(bufs, refs)):
        assert max_rel(_np(b), ref) <= FP32_TOL, i
    assert ks[0] == k0
    assert woq.device_status() == 0


def test_chain_past_its_shared_memory_budget_is_refused():
    w, _, _ = packed_from_weight(workloads.weight(256, 8192, seed=50), 4)
    x = workloads.activations(8, 8192, seed=51).cuda()
    y = torch.full((8, 256), 7.0, device="cuda")
    with pytest.raises(woq.WoqError) as e:
        woq.qgemv_chain([woq.ChainItem(w, x, y)], woq.chain_workspace())
    assert e.value.status == -2
    assert torch.all(y == 7.0)
