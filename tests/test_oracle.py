"""Pins of the CPU oracle to facts fixed outside it (CPU only).

Each test checks the oracle against something other than itself: hand-derived
golden fixtures, exact rational brute force, closed forms, invariants of the
definition, or an independent library routine for a special case. Together
they are chosen so that a dropped term, a wrong sign or index, a wrong nibble
order or a transposed operand in the oracle fails at least one of them.
"""

import bisect
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle.woq_ref import fsum_dot
from tests.golden_io import read_kv, read_rows

# ---------------------------------------------------------------------------
# binary16 rounding of the scale
# ---------------------------------------------------------------------------

_FP16_POS = None


def _fp16_grid():
    """All finite non-negative binary16 values as exact Fractions, with bit patterns."""
    global _FP16_POS
    if _FP16_POS is None:
        vals = []
        for b in range(0, 0x7C00):
            e = (b >> 10) & 0x1F
            m = b & 0x3FF
            if e == 0:
                v = Fraction(m, 1 << 24)
            else:
                v = Fraction(1024 + m, 1 << 10) * (Fraction(2) ** (e - 15))
            vals.append(v)
        _FP16_POS = vals
    return _FP16_POS


def _nearest_fp16_bits(v: Fraction) -> int:
    """Exact nearest binary16 (ties to even) of a non-negative rational; -1 if it overflows."""
    grid = _fp16_grid()
    top = grid[-1]
    ulp_top = Fraction(32)  # spacing of the top binade [32768, 65536)
    if v >= top + ulp_top / 2:
        return -1                         # the midpoint 65520 ties to even, i.e. to infinity
    i = bisect.bisect_left(grid, v)
    if i < len(grid) and grid[i] == v:
        return i
    if i == len(grid):
        return len(grid) - 1
    lo, hi = i - 1, i
    dlo, dhi = v - grid[lo], grid[hi] - v
    if dlo < dhi:
        return lo
    if dhi < dlo:
        return hi
    return lo if lo % 2 == 0 else hi


def test_fp16_round_is_exact_nearest_even():
    rng = np.random.default_rng(11)
    a = np.concatenate([
        rng.uniform(0, 0.2, 400),
        rng.uniform(0, 1e-5, 100),          # subnormal scales
        rng.uniform(0, 458000.0, 100),       # near the top of the range
    ]).astype(np.float32)
    for qmax in (7, 127):
        got = oracle.fp16_round(a.astype(np.float64) / qmax)
        for ai, g in zip(a, got):
            want = _nearest_fp16_bits(Fraction(float(ai)) / qmax)
            assert want >= 0
            assert int(g) == want, (float(ai), qmax, hex(int(g)), hex(want))


def test_fp16_round_agrees_with_struct_half_pack():
    rng = np.random.default_rng(12)
    v = rng.uniform(-70000, 70000, 2000) * np.exp(rng.uniform(-30, 0, 2000))
    got = oracle.fp16_round(v)
    want = np.array([struct.unpack("<H", struct.pack("<e", float(x)))[0] for x in v], dtype=np.uint16)
    np.testing.assert_array_equal(got, want)


def test_fp16_round_ties_to_even_at_exact_midpoints():
    grid = _fp16_grid()
    for b in (0x3092, 0x2008, 0x3C00, 0x0001, 0x03FF, 0x7BFE):
        mid = (grid[b] + grid[b + 1]) / 2
        want = b if b % 2 == 0 else b + 1
        assert int(oracle.fp16_round(np.float64(mid))) == want


def test_scale_closed_forms():
    for row in read_rows("scale_closed_form.txt"):
        bits, a = int(row[0]), float(row[1])
        W = np.zeros((1, 32), dtype=np.float32)
        W[0, 0] = a
        if row[2] == "overflow":
            with pytest.raises(OverflowError):
                oracle.quantise(W, bits)
            continue
        q, sb = oracle.quantise(W, bits)
        assert int(sb[0, 0]) == int(row[2], 16)
        assert oracle.fp16_bits_to_float(sb)[0, 0] == float(row[3])
        W_hat = oracle.dequantise(q, sb)
        assert W_hat[0, 0] == float(row[4])


# ---------------------------------------------------------------------------
# the quantiser: exact brute force over every code
# ---------------------------------------------------------------------------

def _brute_codes(w_row, s_value, bits):
    qmin, qmax = oracle.qrange(bits)
    s = Fraction(float(s_value))
    out = []
    for w in w_row:
        if s == 0:
            out.append(0)
            continue
        wf = Fraction(float(w))
        best, bestd = None, None
        for c in range(qmin, qmax + 1):
            d = abs(wf - s * c)
            if bestd is None or d < bestd or (d == bestd and c % 2 == 0):
                best, bestd = c, d
        out.append(best)
    return out


@pytest.mark.parametrize("bits", [4, 5, 8])
def test_quantiser_matches_brute_force(bits):
    rng = np.random.default_rng(100 + bits)
    W = (rng.standard_normal((3, 96)) * 0.02).astype(np.float32)
    W[1, 32:64] = 0.0                                  # an all-zero block
    W[2, 64:96] = rng.integers(-3, 4, 32).astype(np.float32) * 0.25   # many exact ties
    q, sb = oracle.quantise(W, bits)
    s = oracle.fp16_bits_to_float(sb)
    qmin, qmax = oracle.qrange(bits)
    for n in range(W.shape[0]):
        for j in range(W.shape[1] // 32):
            blk = W[n, 32 * j:32 * j + 32]
            a = max(abs(Fraction(float(v))) for v in blk)
            assert int(sb[n, j]) == max(_nearest_fp16_bits(a / qmax), 0)
            assert list(q[n, 32 * j:32 * j + 32]) == _brute_codes(blk, s[n, j], bits)


def test_ties_round_half_even_golden():
    g = read_kv("ties_int4.txt")
    w = np.array([float(v) for v in g["w"]], dtype=np.float32)[None, :]
    assert w.shape == (1, 32)
    q, sb = oracle.quantise(w, 4)
    assert list(q[0]) == [int(v) for v in g["q"]]
    assert int(sb[0, 0]) == int(g["scale"][0], 16)
    assert list(oracle.pack(q, 4)[0]) == [int(b, 16) for b in g["bytes"]]
    y = oracle.qgemv_ref(np.ones((1, 32), dtype=np.float32), oracle.pack(q, 4), sb, 4)
    assert y[0, 0] == float(g["y_ones"][0])


@pytest.mark.parametrize("bits,name", [(4, "roundtrip_int4.txt"), (5, "roundtrip_int5.txt"),
                                       (8, "roundtrip_int8.txt")])
def test_integer_round_trip_golden(bits, name):
    g = read_kv(name)
    w = np.array([float(v) for v in g["w"]], dtype=np.float32)[None, :]
    assert w.shape == (1, 32)
    q, sb = oracle.quantise(w, bits)
    assert int(sb[0, 0]) == int(g["scale"][0], 16)
    np.testing.assert_array_equal(q[0], w[0].astype(np.int32))
    packed = oracle.pack(q, bits)
    assert list(packed[0]) == [int(b, 16) for b in g["bytes"]]
    np.testing.assert_array_equal(oracle.unpack(packed, bits, 32), q)
    x = np.arange(1, 33, dtype=np.float32)[None, :]
    assert oracle.qgemv_ref(x, packed, sb, bits)[0, 0] == float(g["y_iota"][0])


def test_two_blocks_use_their_own_scales():
    """A row of two blocks with different scales (2 and 1), x = 1..64."""
    t = read_kv("ties_int4.txt")
    r = read_kv("roundtrip_int4.txt")
    w = np.array([float(v) for v in t["w"]] + [float(v) for v in r["w"]], dtype=np.float32)[None, :]
    q, sb = oracle.quantise(w, 4)
    assert [int(v) for v in sb[0]] == [0x4000, 0x3C00]
    x = np.arange(1, 65, dtype=np.float32)[None, :]
    q_t = [int(v) for v in t["q"]]
    w_r = [int(v) for v in r["w"]]
    want = 2 * sum((k + 1) * q_t[k] for k in range(32)) + sum((k + 33) * w_r[k] for k in range(32))
    assert oracle.qgemv_ref(x, oracle.pack(q, 4), sb, 4)[0, 0] == want


@pytest.mark.parametrize("bits", [4, 8])
def test_pack_unpack_is_a_bijection_on_all_bytes(bits):
    allb = np.arange(256, dtype=np.uint8)[None, :]
    K = 256 * 8 // bits
    q = oracle.unpack(allb, bits, K)
    qmin, qmax = oracle.qrange(bits)
    assert q.min() == qmin and q.max() == qmax
    np.testing.assert_array_equal(oracle.pack(q, bits), allb)


def test_int5_pack_unpack_is_a_bijection_on_all_bytes():
    """Every bit of a 20-byte int5 block belongs to exactly one code: any bytes unpack to codes
    that pack back to the same bytes, and every code -16..15 occurs."""
    rng = np.random.default_rng(5)
    b = rng.integers(0, 256, (64, 40)).astype(np.uint8)   # 64 rows of two blocks
    q = oracle.unpack(b, 5, 64)
    assert q.min() == -16 and q.max() == 15
    np.testing.assert_array_equal(oracle.pack(q, 5), b)


@pytest.mark.parametrize("e,bit", [(0, 0), (1, 4), (2, 8), (3, 12), (4, 16), (7, 28), (8, 1),
                                   (12, 17), (29, 23), (31, 31)])
def test_int5_high_bit_positions(e, bit):
    """A block whose only nonzero code is -16 (low bits 0000, bit 4 set) at element e: the
    nibble plane is zero and the high-bit word has exactly the hand-derived bit set."""
    q = np.zeros((1, 32), dtype=np.int32)
    q[0, e] = -16
    p = oracle.pack(q, 5)
    assert not p[0, :16].any()
    word = int.from_bytes(bytes(p[0, 16:20]), "little")
    assert word == 1 << bit


@pytest.mark.parametrize("e,bit", [(0, 0), (3, 12), (4, 16), (8, 1), (29, 23), (31, 31)])
def test_int5_high_bit_position_function(e, bit):
    """The position function itself, on the hand-derived table above (element e of a block:
    bit e/8 + 4(e%4) + 16((e%8)/4) of the high-bit word)."""
    assert oracle.int5_high_bit_position(e) == bit


def test_int5_high_bit_positions_cover_the_word_once():
    assert sorted(oracle.int5_high_bit_position(e) for e in range(32)) == list(range(32))


@pytest.mark.parametrize("bits,K,expect", [(4, 1024, 512), (5, 1024, 640), (8, 1024, 1024),
                                           (4, 32, 16), (5, 128, 80), (8, 96, 96)])
def test_row_bytes_is_the_packed_row_length(bits, K, expect):
    assert oracle.row_bytes(K, bits) == expect
    q = np.zeros((3, K), dtype=np.int32)
    assert oracle.pack(q, bits).shape == (3, expect)


# ---------------------------------------------------------------------------
# special matrices, invariants, linearity, error bound
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [4, 5, 8])
def test_zero_matrix(bits):
    W = np.zeros((5, 64), dtype=np.float32)
    q, sb = oracle.quantise(W, bits)
    assert not sb.any() and not q.any()
    assert not oracle.pack(q, bits).any()
    x = np.random.default_rng(0).standard_normal((3, 64)).astype(np.float32)
    assert not oracle.qgemv_ref(x, oracle.pack(q, bits), sb, bits).any()


@pytest.mark.parametrize("bits,diag,sbits", [(4, 1 - 2.0 ** -12, 0x3092), (5, 1 - 2.0 ** -12, 0x2C44),
                                             (8, 1 - 2.0 ** -14, 0x2008)])
def test_identity(bits, diag, sbits):
    K = 64
    W = np.eye(K, dtype=np.float32)
    q, sb = oracle.quantise(W, bits)
    for n in range(K):
        for j in range(K // 32):
            assert int(sb[n, j]) == (sbits if n // 32 == j else 0)
    x = np.random.default_rng(1).standard_normal((4, K)).astype(np.float32)
    y = oracle.qgemv_ref(x, oracle.pack(q, bits), sb, bits)
    np.testing.assert_array_equal(y, x.astype(np.float64) * diag)


@pytest.mark.parametrize("bits", [4, 5, 8])
def test_invariants(bits):
    rng = np.random.default_rng(7 + bits)
    W = (rng.standard_normal((16, 256)) * 0.02).astype(np.float32)
    q, sb = oracle.quantise(W, bits)
    s = np.repeat(oracle.fp16_bits_to_float(sb), 32, axis=1)
    W_hat = oracle.dequantise(q, sb)
    # |W - W_hat| <= s/2 elementwise (no element is clamped)
    assert np.all(np.abs(W.astype(np.float64) - W_hat) <= s / 2)
    qmin, qmax = oracle.qrange(bits)
    # every nonzero block reaches qmax in magnitude, and never emits qmin
    blk = np.abs(q).reshape(16, -1, 32).max(axis=2)
    assert np.all(blk == qmax)
    assert q.min() > qmin
    # the code keeps the sign of w or is zero
    assert np.all((np.sign(q) == np.sign(W)) | (q == 0))


@pytest.mark.parametrize("bits", [4, 5, 8])
def test_error_bound_against_unquantised_matmul(bits):
    rng = np.random.default_rng(21 + bits)
    W = (rng.standard_normal((24, 128)) * 0.02).astype(np.float32)
    X = rng.standard_normal((5, 128)).astype(np.float32)
    q, sb = oracle.quantise(W, bits)
    y = oracle.qgemv_ref(X, oracle.pack(q, bits), sb, bits)
    exact = X.astype(np.float64) @ W.astype(np.float64).T
    s = np.repeat(oracle.fp16_bits_to_float(sb), 32, axis=1)
    bound = np.abs(X.astype(np.float64)) @ (s / 2).T
    assert np.all(np.abs(y - exact) <= bound * (1 + 1e-12) + 1e-300)
    # and the bound is not vacuous: quantisation error is visible
    assert np.max(np.abs(y - exact)) > 0


def test_linearity_in_x():
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((32, 96)) * 0.02).astype(np.float32)
    q, sb = oracle.quantise(W, 4)
    p = oracle.pack(q, 4)
    x1 = rng.standard_normal((2, 96))
    x2 = rng.standard_normal((2, 96))
    a, b = 0.375, -1.75
    lhs = oracle.qgemv_ref(a * x1 + b * x2, p, sb, 4)
    rhs = a * oracle.qgemv_ref(x1, p, sb, 4) + b * oracle.qgemv_ref(x2, p, sb, 4)
    assert np.max(np.abs(lhs - rhs)) <= 1e-12 * np.max(np.abs(rhs))


def test_matmul_matches_correctly_rounded_sums():
    """Non-square, so a transposed operand fails; fsum of exact products is the truth."""
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((3, 64)) * 0.02).astype(np.float32)
    X = rng.standard_normal((2, 64)).astype(np.float32)
    for bits in (4, 8):
        q, sb = oracle.quantise(W, bits)
        W_hat = oracle.dequantise(q, sb)
        y = oracle.qgemv_ref(X, oracle.pack(q, bits), sb, bits)
        assert y.shape == (2, 3)
        for m in range(2):
            for n in range(3):
                want = fsum_dot(X[m].astype(np.float64), W_hat[n])
                assert abs(y[m, n] - want) <= 4 * 2.0 ** -52 * np.sum(np.abs(X[m] * W_hat[n]))


def test_input_errors():
    with pytest.raises(ValueError):
        oracle.quantise(np.zeros((2, 48), dtype=np.float32), 4)
    with pytest.raises(ValueError):
        W = np.zeros((2, 32), dtype=np.float32)
        W[1, 3] = np.inf
        oracle.quantise(W, 8)
    with pytest.raises(ValueError):
        oracle.qrange(6)
    with pytest.raises(TypeError):
        oracle.quantise(np.zeros((2, 32), dtype=np.float64), 4)


# ---------------------------------------------------------------------------
# the bf16 reading of the tensor-core path
# ---------------------------------------------------------------------------

def test_bf16_round_closed_forms():
    cases = {
        1.0 + 2.0 ** -8: 1.0,                      # tie -> even (mantissa 0)
        1.0 + 3 * 2.0 ** -8: 1.0 + 2.0 ** -6,      # tie -> even (mantissa 2)
        1.0 + 2.0 ** -8 + 2.0 ** -20: 1.0 + 2.0 ** -7,
        -(1.0 + 3 * 2.0 ** -8): -(1.0 + 2.0 ** -6),
        0.142822265625: 0.142578125,               # fp16(1/7) rounded to 8 significant bits
        0.0: 0.0,
        255.0: 255.0,
        257.0: 256.0,
    }
    for v, want in cases.items():
        assert float(oracle.bf16_round(np.float64(v))) == want, v


def test_bf16_round_agrees_with_torch_conversion():
    rng = np.random.default_rng(9)
    v = (rng.standard_normal(20000) * np.exp(rng.uniform(-40, 40, 20000))).astype(np.float32)
    want = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.bf16_round(v.astype(np.float64)), want)


def test_bf16_reading_is_exact_on_bf16_representable_inputs():
    g = read_kv("roundtrip_int8.txt")
    w = np.array([[float(v) for v in g["w"]]] * 3, dtype=np.float32)
    q, sb = oracle.quantise(w, 8)
    p = oracle.pack(q, 8)
    X = np.random.default_rng(4).integers(-100, 100, (4, 32)).astype(np.float32)
    np.testing.assert_array_equal(oracle.qgemm_bf16_ref(X, p, sb, 8), oracle.qgemv_ref(X, p, sb, 8))


def test_bf16_reading_error_is_within_the_tolerance_budget():
    """The reading's own distance from the exact product stays well inside 1e-2 Frobenius."""
    rng = np.random.default_rng(10)
    W = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    X = rng.standard_normal((16, 256)).astype(np.float32)
    for bits in (4, 8):
        q, sb = oracle.quantise(W, bits)
        p = oracle.pack(q, bits)
        e = oracle.qgemm_bf16_ref(X, p, sb, bits) - oracle.qgemv_ref(X, p, sb, bits)
        rel = np.linalg.norm(e) / np.linalg.norm(oracle.qgemv_ref(X, p, sb, bits))
        assert 1e-4 < rel < 1e-2


# ---- greedy pick (qgemv_argmax reference) ----

def test_greedy_ref_first_index_among_ties_and_nan():
    Y = np.array([[1.0, 3.0, 3.0, -2.0],
                  [-5.0, -1.0, -1.0, -7.0],
                  [0.0, np.nan, 9.0, np.nan],
                  [2.0, 2.0, 2.0, 2.0]])
    idx, val = oracle.greedy_ref(Y)
    assert idx.tolist() == [1, 1, 1, 0]
    assert val[0] == 3.0 and val[1] == -1.0 and np.isnan(val[2]) and val[3] == 2.0


def test_qgemv_argmax_ref_on_a_hand_built_weight():
    # every block's max |w| is 7 = qmax for int4, so every scale is exactly 1 and the codes
    # equal the weights; y_j = c_j * x_0 with c = (1, 7, -7, 7, 3) (x_1 = 0)
    K = 32
    W = np.zeros((5, K), dtype=np.float32)
    W[:, 0] = [1.0, 7.0, -7.0, 7.0, 3.0]
    W[:, 1] = 7.0
    q, s = oracle.quantise(W, 4)
    assert np.all(oracle.fp16_bits_to_float(s) == 1.0)
    p = oracle.pack(q, 4)
    x = np.zeros((1, K), dtype=np.float32); x[0, 0] = 2.0
    idx, val = oracle.qgemv_argmax_ref(x, p, s, 4)
    assert idx.tolist() == [1] and val.tolist() == [14.0]   # tie with j = 3: first index
    x[0, 0] = -2.0                                            # now -7 * -2 = 14 at j = 2
    idx, val = oracle.qgemv_argmax_ref(x, p, s, 4)
    assert idx.tolist() == [2] and val.tolist() == [14.0]


# ---- SwiGLU (qgemv_swiglu reference) ----

def test_silu_ref_invariants():
    g = np.array([-700.0, -30.0, -2.5, -1e-3, 0.0, 1e-3, 0.7, 2.5, 30.0, 700.0])
    s = oracle.silu_ref(g)
    assert s[4] == 0.0
    # silu(g) - silu(-g) = g (sigmoid(g) + sigmoid(-g) = 1)
    assert np.allclose(s - oracle.silu_ref(-g), g, rtol=0, atol=1e-12 * np.maximum(1, np.abs(g)))
    # limits: silu(g) -> g for large g, -> 0 for large negative g
    assert s[-1] == 700.0 and s[-2] == pytest.approx(30.0, rel=1e-12)
    assert abs(s[0]) < 1e-300 and abs(s[1]) < 30.0 * 1e-12
    # slope 1/2 at 0: silu(h) / h -> 1/2
    assert s[5] / 1e-3 == pytest.approx(0.5, rel=1e-3)
    assert np.all(np.isfinite(s))


def test_swiglu_ref_pairs_gate_and_up_rows():
    # gate rows (even) and up rows (odd) built so that gate outputs are 0 or large
    K = 32
    W = np.zeros((4, K), dtype=np.float32)
    W[0, :] = 0.0            # gate 0: output 0 -> silu 0
    W[1, 0] = 7.0; W[1, 1] = 7.0   # up 0
    W[2, 0] = 7.0; W[2, 1] = 7.0   # gate 1: output 7 * (x0 + x1)
    W[3, 0] = -7.0; W[3, 1] = 7.0  # up 1: 7 * (x1 - x0)
    q, s = oracle.quantise(W, 4)
    p = oracle.pack(q, 4)
    x = np.zeros((1, K), dtype=np.float32); x[0, 0] = 3.0; x[0, 1] = 5.0
    y = oracle.swiglu_ref(x, p, s, 4)
    assert y.shape == (1, 2)
    assert y[0, 0] == 0.0
    g, u = 7.0 * 8.0, 7.0 * 2.0
    assert y[0, 1] == pytest.approx(oracle.silu_ref(np.array(g))[()] * u, rel=1e-15)
    assert y[0, 1] == pytest.approx(g * u, rel=1e-20)  # sigmoid(56) is 1 to double precision


def test_residual_ref_adds_the_projection_to_the_stream():
    # W = 0 leaves the stream as it is; a one-hot weight row adds one x column, exactly
    K = 64
    rng = np.random.default_rng(3)
    R = rng.standard_normal((3, 5))
    X = rng.standard_normal((3, K)).astype(np.float32)
    q, s = oracle.quantise(np.zeros((5, K), dtype=np.float32), 4)
    assert np.array_equal(oracle.residual_ref(X, oracle.pack(q, 4), s, 4, R), R)
    W = np.zeros((5, K), dtype=np.float32)
    W[2, 7] = 7.0  # block max 7 -> scale 1, code 7
    q, s = oracle.quantise(W, 4)
    Y = oracle.residual_ref(X, oracle.pack(q, 4), s, 4, R)
    want = R.copy()
    want[:, 2] += 7.0 * X[:, 7].astype(np.float64)
    assert np.array_equal(Y, want)
