"""The WOQC weight container: round trip, alignment, checksums, malformed files (CPU only)."""

import numpy as np
import pytest
import torch

import weight_only_bit_qgemv_b200 as woq
from weight_only_bit_qgemv_b200 import container, workloads


def _weights():
    out = {}
    for name, (n, k, bits) in {"layers.0.qkv": (96, 64, 4), "layers.0.down": (40, 160, 8),
                               "layers.0.o5": (33, 256, 5), "lm_head": (7, 32, 8)}.items():
        p, s = woq.qpack(workloads.weight(n, k, seed=n + k), bits)
        out[name] = woq.PackedWeight(p, s, bits, n, k)
    return out


def test_round_trip_is_bit_exact(tmp_path):
    ws = _weights()
    path = str(tmp_path / "m.woqc")
    container.save(path, ws)
    back = container.load(path, device="cpu")
    assert list(back) == list(ws)
    for name, w in ws.items():
        b = back[name]
        assert (b.bits, b.n, b.k) == (w.bits, w.n, w.k)
        assert torch.equal(b.packed, w.packed) and torch.equal(b.scales, w.scales)
        assert b.packed.dtype == torch.uint8 and b.scales.dtype == torch.int16


def test_every_array_starts_on_a_64_byte_boundary_and_holds_the_packed_bytes(tmp_path):
    ws = _weights()
    path = str(tmp_path / "m.woqc")
    container.save(path, ws)
    raw = np.fromfile(path, dtype=np.uint8)
    assert raw[:4].tobytes() == b"WOQC"
    for e in container.read_table(path):
        assert e["off_packed"] % 64 == 0 and e["off_scales"] % 64 == 0
        w = ws[e["name"]]
        got = raw[e["off_packed"]:e["off_packed"] + e["bytes_packed"]]
        assert np.array_equal(got, w.packed.numpy().reshape(-1))
        got_s = raw[e["off_scales"]:e["off_scales"] + e["bytes_scales"]].view(np.uint16)
        assert np.array_equal(got_s, w.scales.numpy().view(np.uint16).reshape(-1))


def test_corrupted_data_is_refused_unless_unchecked(tmp_path):
    path = str(tmp_path / "m.woqc")
    container.save(path, _weights())
    e = container.read_table(path)[1]
    with open(path, "r+b") as f:
        f.seek(e["off_packed"] + 5)
        b = f.read(1)
        f.seek(e["off_packed"] + 5)
        f.write(bytes([b[0] ^ 0x10]))
    with pytest.raises(container.ContainerError):
        container.load(path, device="cpu")
    assert e["name"] in container.load(path, device="cpu", verify=False)


def test_malformed_files_are_refused(tmp_path):
    path = str(tmp_path / "m.woqc")
    container.save(path, _weights())
    data = open(path, "rb").read()
    bad = tmp_path / "bad.woqc"
    bad.write_bytes(b"MQF1" + data[4:])
    with pytest.raises(container.ContainerError):
        container.read_table(str(bad))
    bad.write_bytes(data[:-64])  # last array cut short
    with pytest.raises(container.ContainerError):
        container.read_table(str(bad))
    bad.write_bytes(data[:40])
    with pytest.raises(container.ContainerError):
        container.read_table(str(bad))
    with pytest.raises(ValueError):
        container.save(str(tmp_path / "x.woqc"), {"n" * 64: _weights()["lm_head"]})


@pytest.mark.gpu
def test_loaded_weights_multiply_like_the_originals(tmp_path):
    ws = _weights()
    path = str(tmp_path / "m.woqc")
    container.save(path, ws)
    back = container.load(path, device="cuda")
    for name, w in ws.items():
        x = workloads.activations(3, w.k, seed=1).cuda()
        assert torch.equal(woq.qgemv(x, back[name]), woq.qgemv(x, w.to("cuda")))
