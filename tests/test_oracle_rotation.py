"""Pins the oracle's rotations.

Hadamard (block-diagonal Walsh-Hadamard, "SAW-INT4" Summary/Method and the
UltraQuant method section): the Sylvester matrix from its textbook recursion
(golden fixture), H H^T = b I in integers, the binary32 butterflies equal the
integer matrix product exactly on small integers, R e_i = column i / sqrt(b),
R R = I and norm preservation within binary32 rounding, the scale constant is
the binary32 value nearest 1/sqrt(b) (exact rational check), b = 1 is the
identity, and blocks act independently.

Quaternion (IsoQuant Abstract, T(v) = qL v conj(qR)): Hamilton's unit table
(golden fixture), the 4x4 left-multiplication matrix, the norm identity,
identity quaternions give the identity, T is in SO(4), and the inverse map
undoes it.
"""

from fractions import Fraction

import numpy as np
import pytest

import oracle
from bit_rotated_kv_block_b200 import workloads
from conftest import read_golden_rows


def sylvester(b):
    """Textbook recursion H_1 = [1], H_2n = [[H, H], [H, -H]] in integers."""
    H = np.array([[1]], np.int64)
    while H.shape[0] < b:
        H = np.block([[H, H], [H, -H]])
    return H


def popcount_matrix(b):
    i = np.arange(b)[:, None]
    j = np.arange(b)[None, :]
    par = np.vectorize(lambda n: bin(int(n)).count("1") & 1)(i & j)
    return np.where(par == 1, -1, 1).astype(np.int64)


def test_sylvester_golden_and_popcount_form():
    g = np.array(read_golden_rows("sylvester_h8.txt"), np.int64)
    assert np.array_equal(sylvester(8), g)
    for b in (1, 2, 4, 8, 16, 32, 64, 128, 256):
        assert np.array_equal(sylvester(b), popcount_matrix(b))


@pytest.mark.parametrize("b", [2, 4, 8, 16, 32, 64, 128, 256])
def test_hadamard_orthogonality_integer(b):
    H = sylvester(b)
    assert np.array_equal(H @ H.T, b * np.eye(b, dtype=np.int64))


@pytest.mark.parametrize("b", [2, 4, 8, 16, 32, 64, 128, 256])
def test_fwht_butterflies_equal_integer_product(b):
    rng = np.random.default_rng(b)
    H = sylvester(b)
    for _ in range(20):
        x = rng.integers(-256, 257, size=b)
        got = oracle.fwht_unscaled(x.astype(np.float32))
        # |sum| <= 256 * 256 = 2^16: every partial sum is exact in binary32
        assert np.array_equal(got.astype(np.int64), H @ x)


def test_fwht_unit_vectors_give_golden_columns():
    g = np.array(read_golden_rows("sylvester_h8.txt"), np.int64)
    for j in range(8):
        e = np.zeros(8, np.float32)
        e[j] = 1
        assert np.array_equal(oracle.fwht_unscaled(e).astype(np.int64), g[:, j])


@pytest.mark.parametrize("b", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_hadamard_scale_is_nearest_binary32(b):
    c = oracle.hadamard_scale(b)
    cf = Fraction(float(np.float32(c)))
    # ulp of c in binary32
    m, e = np.frexp(np.float32(c))
    ulp = Fraction(2) ** (int(e) - 24)
    lo, hi = cf - ulp / 2, cf + ulp / 2
    target_sq = Fraction(1, b)  # (1/sqrt(b))^2
    assert lo * lo < target_sq < hi * hi
    bits = int(np.float32(c).view(np.uint32))
    expect = {32: 0x3E3504F3, 128: 0x3DB504F3}
    if b in expect:
        assert bits == expect[b]


@pytest.mark.parametrize("d,b", [(128, 16), (128, 32), (128, 64), (128, 128), (256, 256),
                                 (256, 64), (64, 64)])
def test_hadamard_rotation_matrix_properties(d, b):
    # R applied to the identity gives R's columns: R e_i = H[:, i] / sqrt(b)
    I = np.eye(d, dtype=np.float32)
    Rt = oracle.rotate_f32(I, oracle.ROT_HADAMARD, b)      # row i = R e_i
    R = Rt.T.astype(np.float64)
    ref = np.zeros((d, d))
    for t in range(0, d, b):
        ref[t:t + b, t:t + b] = sylvester(b) / np.sqrt(b)
    assert np.max(np.abs(R - ref)) <= 2 ** -24 / np.sqrt(b) * 1.01
    # R R = I (R symmetric and involutory) within binary32 rounding
    RR = oracle.rotate_f32(Rt, oracle.ROT_HADAMARD, b).astype(np.float64)
    assert np.max(np.abs(RR - np.eye(d))) < 2 * np.log2(max(b, 2)) * 2 ** -24 * 4
    # norms preserved
    x = np.random.default_rng(d + b).standard_normal((64, d)).astype(np.float32)
    y = oracle.rotate_f32(x, oracle.ROT_HADAMARD, b).astype(np.float64)
    n0 = np.linalg.norm(x.astype(np.float64), axis=1)
    assert np.allclose(np.linalg.norm(y, axis=1), n0, rtol=1e-6)
    # double-precision forward equals the explicit matrix
    y64 = oracle.rotate_f64(x, oracle.ROT_HADAMARD, b)
    assert np.allclose(y64, x.astype(np.float64) @ ref.T, atol=1e-12)
    # and its inverse undoes it
    assert np.allclose(oracle.unrotate_f64(y64, oracle.ROT_HADAMARD, b), x, atol=1e-12)


def test_hadamard_block_one_is_identity_and_blocks_independent():
    x = np.random.default_rng(3).standard_normal((8, 128)).astype(np.float32)
    assert np.array_equal(oracle.rotate_f32(x, oracle.ROT_HADAMARD, 1), x)
    y = oracle.rotate_f32(x, oracle.ROT_HADAMARD, 32)
    for t in range(0, 128, 32):
        part = oracle.rotate_f32(np.ascontiguousarray(x[:, t:t + 32]), oracle.ROT_HADAMARD, 32)
        assert np.array_equal(y[:, t:t + 32], part)
    assert np.array_equal(oracle.rotate_f32(x, oracle.ROT_NONE, 0), x)


# ---------------------------------------------------------------- quaternions

UNITS = {"1": [1, 0, 0, 0], "i": [0, 1, 0, 0], "j": [0, 0, 1, 0], "k": [0, 0, 0, 1]}


def test_hamilton_unit_table_golden():
    rows = read_golden_rows("quaternion_table.txt")
    cols = [r[0] for r in rows]          # right factors in the same order as the rows
    assert cols == ["1", "i", "j", "k"]
    for row in rows:
        a = row[0]
        for b, entry in zip(cols, row[1:]):
            sign = -1 if entry.startswith("-") else 1
            expect = sign * np.array(UNITS[entry.lstrip("-")], np.float32)
            got = oracle.hamilton(np.array(UNITS[a], np.float32), np.array(UNITS[b], np.float32))
            assert np.array_equal(got, expect), (a, b)


def left_matrix(a):
    """Textbook matrix of v -> a v for a = (w, x, y, z)."""
    w, x, y, z = a
    return np.array([[w, -x, -y, -z], [x, w, -z, y], [y, z, w, -x], [z, -y, x, w]])


def test_hamilton_matches_matrix_form_and_norms():
    g = np.random.default_rng(7)
    for _ in range(500):
        a = g.standard_normal(4).astype(np.float32)
        b = g.standard_normal(4).astype(np.float32)
        got = oracle.hamilton(a, b).astype(np.float64)
        ref = left_matrix(a.astype(np.float64)) @ b.astype(np.float64)
        scale = np.linalg.norm(a) * np.linalg.norm(b)
        assert np.max(np.abs(got - ref)) <= 4 * 2 ** -24 * scale
        assert abs(np.linalg.norm(got) - scale) <= 8 * 2 ** -24 * scale


def test_quaternion_rotation_properties():
    d = 128
    quat = workloads.random_quaternions(5, d)
    # identity table -> identity map, exactly
    ident = np.zeros((d // 4, 2, 4), np.float32)
    ident[:, :, 0] = 1
    x = np.random.default_rng(11).standard_normal((32, d)).astype(np.float32)
    assert np.array_equal(oracle.rotate_f32(x, oracle.ROT_QUAT, 0, ident), x)
    # norms preserved (unit quaternions rounded to binary32)
    y = oracle.rotate_f32(x, oracle.ROT_QUAT, 0, quat).astype(np.float64)
    n0 = np.linalg.norm(x.astype(np.float64), axis=1)
    assert np.allclose(np.linalg.norm(y, axis=1), n0, rtol=4e-7 * 4)
    # binary32 path agrees with the double-precision map
    y64 = oracle.rotate_f64(x, oracle.ROT_QUAT, 0, quat)
    assert np.max(np.abs(y - y64)) < 1e-5
    # inverse undoes the forward map
    assert np.allclose(oracle.unrotate_f64(y64, oracle.ROT_QUAT, 0, quat), x, atol=1e-12)
    # each 4x4 block is a rotation: orthogonal with determinant +1
    M = oracle.rotate_f64(np.eye(d), oracle.ROT_QUAT, 0, quat).T
    for j in range(d // 4):
        B = M[4 * j:4 * j + 4, 4 * j:4 * j + 4]
        assert np.allclose(B @ B.T, np.eye(4), atol=1e-6)
        assert abs(np.linalg.det(B) - 1) < 1e-6
    # and blocks do not mix
    off = M.copy()
    for j in range(d // 4):
        off[4 * j:4 * j + 4, 4 * j:4 * j + 4] = 0
    assert np.all(off == 0)


def test_quaternion_map_is_left_times_conj_right():
    quat = workloads.random_quaternions(9, 8)
    v = np.random.default_rng(2).standard_normal((1, 8))
    y = oracle.rotate_f64(v, oracle.ROT_QUAT, 0, quat)[0]
    for j in range(2):
        qL = quat[j, 0].astype(np.float64)
        qR = quat[j, 1].astype(np.float64)
        qRc = qR * np.array([1, -1, -1, -1])
        ref = left_matrix(left_matrix(qL) @ v[0, 4 * j:4 * j + 4]) @ qRc
        assert np.allclose(y[4 * j:4 * j + 4], ref, atol=1e-14)
