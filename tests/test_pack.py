"""Host qpack (C++, through the C ABI) is bit-exact with the oracle (CPU only)."""

import numpy as np
import pytest
import torch

import oracle
import weight_only_bit_qgemv_b200 as woq
from weight_only_bit_qgemv_b200 import _lib, workloads
from tests.golden_io import read_kv, read_rows


def _both(W, bits):
    p, s = woq.qpack(torch.from_numpy(W), bits)
    q_ref, s_ref = oracle.quantise(W, bits)
    return p.numpy(), s.numpy().view(np.uint16), oracle.pack(q_ref, bits), s_ref


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("shape", [(1, 32), (3, 96), (37, 1024), (64, 3072)])
def test_random_matches_oracle_bit_exactly(bits, shape):
    W = workloads.weight(*shape, seed=shape[0] * 7 + bits).numpy()
    p, s, p_ref, s_ref = _both(W, bits)
    np.testing.assert_array_equal(s, s_ref)
    np.testing.assert_array_equal(p, p_ref)


@pytest.mark.parametrize("bits", [4, 5, 8])
def test_adversarial_blocks_match_oracle(bits):
    rng = np.random.default_rng(bits)
    W = np.zeros((8, 256), dtype=np.float32)
    W[0] = rng.integers(-6, 7, 256) * 0.5           # exact ties everywhere
    W[1, :32] = 0.0                                  # all-zero block
    W[1, 32:] = rng.standard_normal(224) * 1e-6      # subnormal binary16 scales
    W[2] = rng.standard_normal(256) * 1e-9           # scales that underflow to 0
    W[3] = rng.standard_normal(256) * 3e3            # large values
    W[4] = np.float32(1e-45)                         # float32 subnormal inputs
    W[5, ::2] = 1.0
    W[5, 1::2] = -1.0
    W[6] = rng.standard_normal(256).astype(np.float32)
    W[6, 5] = -np.abs(W[6]).max() * 2               # negative maximum
    W[7] = np.linspace(-1, 1, 256, dtype=np.float32)
    p, s, p_ref, s_ref = _both(W, bits)
    np.testing.assert_array_equal(s, s_ref)
    np.testing.assert_array_equal(p, p_ref)


def test_golden_fixtures_through_the_c_abi():
    g = read_kv("ties_int4.txt")
    w = np.array([[float(v) for v in g["w"]]], dtype=np.float32)
    p, s = woq.qpack(torch.from_numpy(w), 4)
    assert list(p.numpy()[0]) == [int(b, 16) for b in g["bytes"]]
    assert int(s.numpy().view(np.uint16)[0, 0]) == int(g["scale"][0], 16)
    for bits, name in ((4, "roundtrip_int4.txt"), (5, "roundtrip_int5.txt"), (8, "roundtrip_int8.txt")):
        g = read_kv(name)
        w = np.array([[float(v) for v in g["w"]]], dtype=np.float32)
        p, s = woq.qpack(torch.from_numpy(w), bits)
        assert list(p.numpy()[0]) == [int(b, 16) for b in g["bytes"]]
    for row in read_rows("scale_closed_form.txt"):
        bits, a = int(row[0]), float(row[1])
        W = np.zeros((1, 32), dtype=np.float32)
        W[0, 7] = a
        if row[2] == "overflow":
            with pytest.raises(_lib.WoqError) as e:
                woq.qpack(torch.from_numpy(W), bits)
            assert e.value.status == _lib.WOQ_ERANGE
        else:
            _, s = woq.qpack(torch.from_numpy(W), bits)
            assert int(s.numpy().view(np.uint16)[0, 0]) == int(row[2], 16)


def test_errors():
    W = np.zeros((2, 32), dtype=np.float32)
    W[1, 1] = np.nan
    with pytest.raises(_lib.WoqError) as e:
        woq.qpack(torch.from_numpy(W), 4)
    assert e.value.status == _lib.WOQ_ERANGE
    W[1, 1] = -np.inf
    with pytest.raises(_lib.WoqError):
        woq.qpack(torch.from_numpy(W), 8)
    L = _lib.lib()
    buf = np.zeros(64, dtype=np.float32)
    out = np.zeros(64, dtype=np.uint8)
    sc = np.zeros(4, dtype=np.uint16)
    ptr = lambda a: a.ctypes.data
    assert L.qpack(ptr(buf), 1, 48, 4, ptr(out), ptr(sc)) == _lib.WOQ_ESHAPE
    assert L.qpack(ptr(buf), 1, 32, 3, ptr(out), ptr(sc)) == _lib.WOQ_EINVAL
    assert L.qpack(None, 1, 32, 4, ptr(out), ptr(sc)) == _lib.WOQ_EINVAL
    assert L.qpack(ptr(buf), 0, 32, 4, ptr(out), ptr(sc)) == _lib.WOQ_ESHAPE


def test_multithreaded_pack_matches_oracle_on_a_decoder_shape():
    W = workloads.weight(3072, 1024, seed=workloads.layer_seed(0, 4)).numpy()
    for bits in (4, 5, 8):
        p, s, p_ref, s_ref = _both(W, bits)
        np.testing.assert_array_equal(s, s_ref)
        np.testing.assert_array_equal(p, p_ref)
