"""GPU parity of qgemv_chain (a decode step's GEMVs as one persistent launch) against the CPU
oracle, item by item, through the C ABI.

Each item is checked against the oracle applied to the inputs that item actually read (the
GPU's own earlier outputs where the chain feeds one item into the next), at the FP32 paths'
tolerance; the chain's order is checked by feeding outputs forward.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import weight_only_bit_qgemv_b200 as woq
from weight_only_bit_qgemv_b200 import _lib, workloads
from tests.gpu_util import FP32_TOL, max_rel, packed_from_weight, packed_raw

pytestmark = pytest.mark.gpu


def decoder_block(bits, layer=0):
    """qkv [4096x1024], o [1024x2048], gate|up interleaved [6144x1024], down [1024x3072]."""
    ws = [workloads.weight(n, k, seed=workloads.layer_seed(layer, i))
          for i, (_, n, k) in enumerate(workloads.DECODER_PROJ)]
    qkv = torch.cat(ws[0:3], 0)
    gu = woq.interleave_rows(ws[4], ws[5])
    return [packed_from_weight(W, bits) for W in (qkv, ws[3], gu, ws[6])]


def np_(t):
    return t.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("m", [1, 2, 3, 4, 8])
def test_decoder_block_chain(bits, m):
    """x0 -> qkv; attn -> o + h0 -> h1; h1 -> gate|up SwiGLU -> a; a -> down + h1 -> h2."""
    (wq, pq, sq), (wo, po, so), (wg, pg, sg), (wd, pd, sd) = decoder_block(bits)
    x0 = workloads.activations(m, 1024, seed=1).cuda()
    attn = workloads.activations(m, 2048, seed=2).cuda()
    h0 = workloads.activations(m, 1024, seed=3).cuda()
    y_qkv = torch.full((m, 4096), float("nan"), device="cuda")
    h1 = torch.full((m, 1024), float("nan"), device="cuda")
    a = torch.full((m, 3072), float("nan"), device="cuda")
    h2 = torch.full((m, 1024), float("nan"), device="cuda")
    ws = woq.chain_workspace()
    woq.qgemv_chain([woq.ChainItem(wq, x0, y_qkv),
                     woq.ChainItem(wo, attn, h1, h0, "residual"),
                     woq.ChainItem(wg, h1, a, None, "swiglu"),
                     woq.ChainItem(wd, a, h2, h1, "residual")], ws)
    torch.cuda.synchronize()
    assert max_rel(np_(y_qkv), oracle.qgemv_ref(np_(x0), pq, sq, bits)) <= FP32_TOL
    assert max_rel(np_(h1), oracle.residual_ref(np_(attn), po, so, bits, np_(h0))) <= FP32_TOL
    assert max_rel(np_(a), oracle.swiglu_ref(np_(h1), pg, sg, bits)) <= FP32_TOL
    assert max_rel(np_(h2), oracle.residual_ref(np_(a), pd, sd, bits, np_(h1))) <= FP32_TOL
    assert torch.count_nonzero(ws).item() == 0  # counters reset for the next call
    assert woq.device_status() == 0


def test_in_place_residual_stream_and_repeat_calls_are_bit_identical():
    """The residual stream h updated in place twice (o, then down through the SwiGLU); three
    calls from the same inputs give the same bits."""
    (wq, _, _), (wo, po, so), (wg, pg, sg), (wd, pd, sd) = decoder_block(4, layer=3)
    attn = workloads.activations(1, 2048, seed=5).cuda()
    h_init = workloads.activations(1, 1024, seed=6).cuda()
    a = torch.empty(1, 3072, device="cuda")
    ws = woq.chain_workspace()
    outs = []
    for _ in range(3):
        h = h_init.clone()
        woq.qgemv_chain([woq.ChainItem(wo, attn, h, h, "residual"),
                         woq.ChainItem(wg, h, a, None, "swiglu"),
                         woq.ChainItem(wd, a, h, h, "residual")], ws)
        outs.append((h.clone(), a.clone()))
    torch.cuda.synchronize()
    h1 = oracle.residual_ref(np_(attn), po, so, 4, np_(h_init))
    a_ref = oracle.swiglu_ref(h1, pg, sg, 4)
    assert max_rel(np_(outs[0][1]), a_ref) <= FP32_TOL
    h2 = oracle.residual_ref(np_(outs[0][1]), pd, sd, 4, h1)
    assert max_rel(np_(outs[0][0]), h2) <= FP32_TOL
    for h, aa in outs[1:]:
        assert torch.equal(h, outs[0][0]) and torch.equal(aa, outs[0][1])


@pytest.mark.parametrize("bits", [4, 8])
def test_ragged_and_tiny_items_every_code(bits):
    """n not a multiple of the grid (and below it: most CTAs hold no rows), k = 256..4096,
    random codes (every code, -8 / -128 included)."""
    shapes = [(1000, 256), (33, 1024), (4099, 256), (300, 4096)]
    ws_ = [packed_raw(n, k, bits, seed=n + k) for n, k in shapes]
    m = 3
    x = workloads.activations(m, 256, seed=9).cuda()
    ys = [torch.empty(m, n, device="cuda") for n, _ in shapes]
    x2 = workloads.activations(m, 1024, seed=10).cuda()
    x4 = workloads.activations(m, 4096, seed=11).cuda()
    items = [woq.ChainItem(ws_[0][0], x, ys[0]),
             woq.ChainItem(ws_[1][0], x2, ys[1]),
             woq.ChainItem(ws_[2][0], x, ys[2]),
             woq.ChainItem(ws_[3][0], x4, ys[3])]
    ws = woq.chain_workspace()
    woq.qgemv_chain(items, ws)
    for it, (w, p, s) in zip(items, ws_):
        assert max_rel(np_(it.y), oracle.qgemv_ref(np_(it.x), p, s, bits)) <= FP32_TOL


def test_matches_separate_calls_within_tolerance_and_replays_from_a_graph():
    (wq, pq, sq), (wo, _, _), (wg, _, _), (wd, _, _) = decoder_block(4, layer=7)
    x0 = workloads.activations(1, 1024, seed=12).cuda()
    attn = workloads.activations(1, 2048, seed=13).cuda()
    h0 = workloads.activations(1, 1024, seed=14).cuda()
    bufs = [torch.empty(1, 4096, device="cuda"), torch.empty(1, 1024, device="cuda"),
            torch.empty(1, 3072, device="cuda"), torch.empty(1, 1024, device="cuda")]
    ws = woq.chain_workspace()
    items = [woq.ChainItem(wq, x0, bufs[0]), woq.ChainItem(wo, attn, bufs[1], h0, "residual"),
             woq.ChainItem(wg, bufs[1], bufs[2], None, "swiglu"),
             woq.ChainItem(wd, bufs[2], bufs[3], bufs[1], "residual")]
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        woq.qgemv_chain(items, ws, stream=st)
    st.synchronize()
    ref = [b.clone() for b in bufs]
    sep = [woq.qgemv(x0, wq), woq.qgemv_residual(attn, wo, h0)]
    sep.append(woq.qgemv_swiglu(ref[1], wg))
    sep.append(woq.qgemv_residual(ref[2], wd, ref[1]))
    for a, b in zip(ref, sep):
        assert max_rel(np_(a), np_(b)) <= FP32_TOL
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        woq.qgemv_chain(items, ws, stream=st)
    for b in bufs:
        b.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    for a, b in zip(ref, bufs):
        assert torch.equal(a, b)
    assert torch.count_nonzero(ws).item() == 0


def test_rejects_bad_arguments():
    w, _, _ = packed_raw(256, 512, 4, seed=1)
    w96, _, _ = packed_raw(256, 96, 4, seed=2)
    x = torch.zeros(1, 512, device="cuda")
    y = torch.zeros(1, 256, device="cuda")
    ws = woq.chain_workspace()
    with pytest.raises(woq.WoqError):
        woq.qgemv_chain([woq.ChainItem(w96, torch.zeros(1, 96, device="cuda"), y)], ws)  # k % 256
    with pytest.raises(woq.WoqError):
        woq.qgemv_chain([woq.ChainItem(w, x, y)] * 9, ws)  # more than 8 items
    with pytest.raises(woq.WoqError):
        woq.qgemv_chain([woq.ChainItem(w, torch.zeros(9, 512, device="cuda"), torch.zeros(9, 256, device="cuda"))], ws)
    with pytest.raises(woq.WoqError):
        woq.qgemv_chain([woq.ChainItem(w, x, y)], ws[1:])  # misaligned workspace
    with pytest.raises(woq.WoqError):
        woq.qgemv_chain([woq.ChainItem(w, x, x[:, :256])], ws)  # y overlaps x
    L = _lib.lib()
    assert L.qgemv_chain(None, 1, 1, ws.data_ptr(), 256, None) == _lib.WOQ_EINVAL
    arr = (_lib.WoqChainItem * 1)()
    d = w.desc()
    arr[0].w = ctypes.pointer(d)
    arr[0].x, arr[0].y, arr[0].r, arr[0].epilogue = x.data_ptr(), y.data_ptr(), None, 0
    assert L.qgemv_chain(arr, 1, 1, None, 0, None) == _lib.WOQ_EWORKSPACE
    arr[0].epilogue = 2  # residual without r
    assert L.qgemv_chain(arr, 1, 1, ws.data_ptr(), 256, None) == _lib.WOQ_EINVAL
    assert torch.count_nonzero(ws).item() == 0


def test_waits_that_give_up_are_reported_without_a_hang():
    """The test hook makes every CTA's wait for the others wait for one arrival too many,
    bounded by 100k cycles: the launch returns, woq_device_status reports WOQ_ETIMEOUT, and after
    zeroing the workspace the next call is correct again."""
    (wq, pq, sq), (wo, _, _), (wg, _, _), (wd, _, _) = decoder_block(4, layer=9)
    x0 = workloads.activations(1, 1024, seed=15).cuda()
    y = torch.empty(1, 4096, device="cuda")
    y2 = torch.empty(1, 4096, device="cuda")
    ws = woq.chain_workspace()
    _lib.lib().woq_debug_set_wait_limit(-100000)
    try:
        woq.qgemv_chain([woq.ChainItem(wq, x0, y), woq.ChainItem(wq, x0, y2)], ws)
        assert woq.device_status() == _lib.WOQ_ETIMEOUT
    finally:
        _lib.lib().woq_debug_set_wait_limit(0)
    ws.zero_()
    woq.qgemv_chain([woq.ChainItem(wq, x0, y), woq.ChainItem(wq, x0, y2)], ws)
    torch.cuda.synchronize()
    assert woq.device_status() == _lib.WOQ_OK
    assert max_rel(np_(y2), oracle.qgemv_ref(np_(x0), pq, sq, 4)) <= FP32_TOL
