"""Pins for oracle.encode: encode pipeline and packed layout.

Independent references: a brute-force encoder at d=8 written with explicit loops, the dense
Hadamard matrix from scipy, a dense S, and the nearest-centroid argmin over all 2^b levels
(Lloyd-Max cells are nearest-centroid cells, [LP] 三.4); hand-packed byte examples.
"""
import math

import numpy as np
import pytest
from scipy.linalg import hadamard

from oracle import codebook, encode


def brute_force_encode(x, D, S, c):
    """One vector, explicit loops, dense matrices, argmin over levels."""
    d = len(x)
    nu = math.sqrt(sum(v * v for v in x))
    u = [v / nu for v in x] if nu > 0 else [0.0] * d
    H = hadamard(d)
    y = [sum(H[i][j] * D[j] * u[j] for j in range(d)) / math.sqrt(d) for i in range(d)]
    codes = []
    for yi in y:
        dist = [abs(yi - ck) for ck in c]
        codes.append(int(np.argmin(dist)))
    r = [y[i] - c[codes[i]] for i in range(d)]
    gamma = math.sqrt(sum(v * v for v in r))
    z = [sum(S[i][j] * r[j] for j in range(d)) for i in range(len(S))]
    bits = [1 if zi >= 0 else 0 for zi in z]
    return nu, y, codes, gamma, z, bits


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_encode_matches_brute_force_d8(bits):
    d, m, n = 8, 32, 200
    rng = np.random.default_rng(bits)
    x = rng.standard_normal((n, d)) * rng.lognormal(size=d)
    D = rng.choice([-1.0, 1.0], size=d)
    S = rng.standard_normal((m, d))
    c, t = codebook.codebook(d, bits)
    enc = encode.encode(x, D, S, c, t)
    for i in range(n):
        nu, y, codes, gamma, z, sb = brute_force_encode(x[i].tolist(), D.tolist(), S.tolist(), c.tolist())
        assert enc.norm[i] == pytest.approx(nu, rel=1e-12)
        np.testing.assert_allclose(enc.y[i], y, atol=1e-12)
        assert enc.codes[i].tolist() == codes
        assert enc.rnorm[i] == pytest.approx(gamma, rel=1e-10, abs=1e-13)
        np.testing.assert_allclose(enc.z[i], z, atol=1e-12)
        assert enc.bits[i].tolist() == sb


def test_quantize_tie_goes_to_upper_cell():
    t = np.array([-0.5, 0.0, 0.5])
    y = np.array([-0.5, -0.50000001, 0.0, 0.5, 0.9, -0.9])
    assert encode.quantize(y, t).tolist() == [1, 0, 2, 3, 3, 0]


def test_zero_vector():
    d, m = 16, 32
    rng = np.random.default_rng(0)
    D = rng.choice([-1.0, 1.0], size=d)
    S = rng.standard_normal((m, d))
    c, t = codebook.codebook(d, 2)
    enc = encode.encode(np.zeros((1, d)), D, S, c, t)
    assert enc.norm[0] == 0.0
    # y = 0 lies on the middle threshold 0 and goes to the upper middle cell
    assert enc.codes[0].tolist() == [2] * d


def test_pack_codes_hand_example():
    # d=8, b=2, codes 0,1,2,3,3,2,1,0:
    #   plane 0 (bit 0 of each code) = 0,1,0,1,1,0,1,0 -> LSB-first byte 0b01011010 = 0x5A
    #   plane 1 (bit 1 of each code) = 0,0,1,1,1,1,0,0 -> 0b00111100 = 0x3C
    codes = np.array([[0, 1, 2, 3, 3, 2, 1, 0]])
    buf = encode.pack_codes(codes, 2)
    assert buf.shape == (1, 16)
    assert buf[0].tolist() == [0x5A, 0x3C] + [0] * 14
    np.testing.assert_array_equal(encode.unpack_codes(buf, 8, 2), codes)


def test_pack_codes_plane_offsets_d128():
    # code_j = 5 (binary 101) only at j = 9: plane 0 byte 1 bit 1, plane 2 byte 32 + 1 bit 1
    codes = np.zeros((1, 128), dtype=np.int64)
    codes[0, 9] = 5
    buf = encode.pack_codes(codes, 3)
    assert buf.shape == (1, 48)
    expect = [0] * 48
    expect[1] = 0x02
    expect[32 + 1] = 0x02
    assert buf[0].tolist() == expect


def test_pack_signs_hand_example():
    bits = np.zeros((1, 32), dtype=np.uint8)
    bits[0, [0, 7, 8, 31]] = 1
    buf = encode.pack_signs(bits)
    assert buf.shape == (1, 16)
    assert buf[0, :4].tolist() == [0x81, 0x01, 0x00, 0x80]
    np.testing.assert_array_equal(encode.unpack_signs(buf, 32), bits)


@pytest.mark.parametrize("d,bits", [(8, 1), (8, 3), (16, 2), (32, 4), (128, 2), (128, 3), (1024, 1), (1024, 3)])
def test_pack_round_trip(d, bits):
    rng = np.random.default_rng(d * 10 + bits)
    codes = rng.integers(0, 1 << bits, size=(7, d))
    buf = encode.pack_codes(codes, bits)
    assert buf.shape[1] == encode.code_bytes(d, bits) and buf.shape[1] % 16 == 0
    np.testing.assert_array_equal(encode.unpack_codes(buf, d, bits), codes)


@pytest.mark.parametrize("m", [32, 64, 128, 1024])
def test_sign_round_trip(m):
    rng = np.random.default_rng(m)
    b = rng.integers(0, 2, size=(5, m)).astype(np.uint8)
    buf = encode.pack_signs(b)
    assert buf.shape[1] == encode.sign_bytes(m) and buf.shape[1] % 16 == 0
    np.testing.assert_array_equal(encode.unpack_signs(buf, m), b)


def test_packed_sizes_at_the_configs():
    # codes ceil(b d / 128) * 16 B, signs m/8 B: 2+QJL at d=128 -> 32 + 16, V3 -> 48,
    # d=1024 1+QJL -> 128 + 128
    assert encode.code_bytes(128, 2) == 32 and encode.sign_bytes(128) == 16
    assert encode.code_bytes(128, 3) == 48
    assert encode.code_bytes(1024, 1) == 128 and encode.sign_bytes(1024) == 128
    assert encode.code_bytes(1024, 3) == 384


def test_rotation_removes_outliers_before_quantization():
    # [JJ] 第二部分 第一步: outlier channels (x20) no longer dominate after rotation.
    d = 128
    rng = np.random.default_rng(5)
    x = rng.standard_normal((256, d))
    x[:, :4] *= 20
    D = rng.choice([-1.0, 1.0], size=d)
    c, t = codebook.codebook(d, 2)
    enc = encode.encode(x, D, np.zeros((0, d)), c, t)
    # the rotated unit vectors have coordinates of size ~1/sqrt(d), far below the outlier share
    assert np.max(np.abs(enc.y)) < 0.6
    u = x / np.linalg.norm(x, axis=1, keepdims=True)
    assert np.max(np.abs(u)) > 0.9


def test_block16_layout_hand_example():
    # d=8, b=3: 16 slots; slot 5 has code_2 = 6 (binary 110) and code_3 = 1, all others 0.
    #   W[0*8 + 2]: plane 0 of j=2 is 0, plane 1 is 1 -> bit 16+5
    #   W[0*8 + 3]: plane 0 of j=3 is 1 -> bit 5
    #   plane 2 (odd last plane) of j=2 is 1 -> W[1*8 + 1], bit 16*0 + 5
    codes = np.zeros((16, 8), dtype=np.int64)
    codes[5, 2] = 6
    codes[5, 3] = 1
    buf = encode.pack_codes_block16(codes, 3)
    assert buf.shape == (16, 16)
    words = buf.reshape(-1).view(np.uint32)
    expect = np.zeros(64, dtype=np.uint32)
    expect[2] = 1 << 21
    expect[3] = 1 << 5
    expect[8 + 1] = 1 << 5
    np.testing.assert_array_equal(words, expect)
    np.testing.assert_array_equal(encode.unpack_codes_block16(buf, 8, 3), codes)


@pytest.mark.parametrize("d,bits", [(8, 1), (8, 2), (16, 3), (128, 2), (128, 3), (128, 4), (64, 1)])
def test_block16_round_trip_and_size(d, bits):
    rng = np.random.default_rng(d + bits)
    codes = rng.integers(0, 1 << bits, size=(48, d))
    buf = encode.pack_codes_block16(codes, bits)
    assert buf.shape == (48, encode.code_bytes(d, bits))
    np.testing.assert_array_equal(encode.unpack_codes_block16(buf, d, bits), codes)
    # same information as the row layout: 16 * (b*d/8) meaningful bytes per block
    used = 16 * bits * d // 8
    assert np.all(buf.reshape(3, -1)[:, used:] == 0)


def test_store_norms_half_precision():
    """fp16 norm storage: round to nearest even on the half grid (2^-10 spacing in [1, 2)),
    saturation at the largest half, codes and signs untouched; 32 bits leaves the encoding as is."""
    n = 6
    enc = encode.Encoded(norm=np.array([1.0, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 3.14159, 1e6, 0.0]),
                       codes=np.zeros((n, 4), dtype=np.int64),
                       rnorm=np.array([0.5, 0.25 + 2.0 ** -13, 2.0 ** -14 * 1.5, 70000.0, 1e-3, 0.0]),
                       bits=np.ones((n, 4), dtype=np.uint8), y=np.zeros((n, 4)), z=np.zeros((n, 4)))
    assert encode.store_norms(enc, 32) is enc
    h = encode.store_norms(enc, 16)
    # halfway cases go to the even neighbour: 1 + 2^-11 -> 1, 1 + 3 2^-11 -> 1 + 2^-9
    np.testing.assert_array_equal(h.norm[:3], [1.0, 1.0, 1.0 + 2.0 ** -9])
    # pi on the half grid of [2, 4) (spacing 2^-9): 3.140625 (1608 * 2^-9)
    assert h.norm[3] == 1608 * 2.0 ** -9
    assert h.norm[4] == 65504.0 and h.rnorm[3] == 65504.0
    # 0.25 + 2^-13 is halfway on the [0.25, 0.5) grid (spacing 2^-12): even -> 0.25
    assert h.rnorm[1] == 0.25
    # 1.5 * 2^-14 is a normal half exactly
    assert h.rnorm[2] == 1.5 * 2.0 ** -14
    np.testing.assert_array_equal(h.codes, enc.codes)
    np.testing.assert_array_equal(h.bits, enc.bits)
    with pytest.raises(ValueError):
        encode.store_norms(enc, 8)
