"""Pins the oracle's two further rotation kinds.

* IsoQuant-Fast (page "IsoQuant: Hardware-Aligned SO(4) Isoclinic Rotations
  for LLM KV Cache Compression", Abstract: the variant that keeps one
  isoclinic factor): v -> qL v per 4-channel block. Pinned against the 4x4
  left-multiplication matrix of the quaternion written out from its
  definition, the textbook unit products (i v, j v, k v), exact results for
  Hurwitz quaternions (components +-1/2) on small integers, norm
  preservation and the inverse round trip.
* Randomised-sign Hadamard: channels multiplied by a fixed +-1 table, then the
  block Hadamard rotation. Pinned against the plain Hadamard (all signs +1),
  the Sylvester matrix times the sign diagonal in exact integers, and the
  round trip R^-1 R = I.
"""

import numpy as np
import pytest

import oracle
from bit_rotated_kv_block_b200 import workloads


def left_matrix(q):
    """4x4 matrix of v -> q v for q = (w, x, y, z), from the Hamilton product."""
    w, x, y, z = q
    return np.array([[w, -x, -y, -z],
                     [x, w, -z, y],
                     [y, z, w, -x],
                     [z, -y, x, w]], dtype=np.float64)


def table_from_left(ql):
    """[d/4][2][4] table with the given left factors and identity right ones."""
    t = np.zeros((ql.shape[0], 2, 4), np.float32)
    t[:, 0] = ql
    t[:, 1, 0] = 1.0
    return t


def test_fast_matches_left_multiplication_matrix():
    d = 64
    g = np.random.default_rng(0)
    quat = workloads.random_quaternions(7, d)
    x = g.standard_normal((10, d)).astype(np.float32)
    y = oracle.rotate_f32(x, oracle.ROT_QUAT_FAST, 0, quat)
    for j in range(d // 4):
        M = left_matrix(quat[j, 0].astype(np.float64))
        ref = x[:, 4 * j:4 * j + 4].astype(np.float64) @ M.T
        # four correctly rounded multiply-adds: within 4 binary32 ulps of the
        # largest term's scale
        scale = np.abs(x[:, 4 * j:4 * j + 4]).max(axis=1, keepdims=True)
        assert np.all(np.abs(y[:, 4 * j:4 * j + 4] - ref) <= 4 * 2.0 ** -23 * scale)
    # double precision forward equals the matrix to rounding
    yd = oracle.rotate_f64(x.astype(np.float64), oracle.ROT_QUAT_FAST, 0, quat)
    for j in range(d // 4):
        M = left_matrix(quat[j, 0].astype(np.float64))
        assert np.allclose(yd[:, 4 * j:4 * j + 4], x[:, 4 * j:4 * j + 4].astype(np.float64) @ M.T,
                           rtol=0, atol=1e-12)


def test_fast_unit_products_and_identity():
    d = 16
    v = np.arange(1, d + 1, dtype=np.float32)[None]
    units = {"1": [1, 0, 0, 0], "i": [0, 1, 0, 0], "j": [0, 0, 1, 0], "k": [0, 0, 0, 1]}
    out = {}
    for name, q in units.items():
        t = table_from_left(np.tile(np.array(q, np.float32), (d // 4, 1)))
        out[name] = oracle.rotate_f32(v, oracle.ROT_QUAT_FAST, 0, t)[0].reshape(-1, 4)
    w, x, y, z = v[0].reshape(-1, 4).T
    assert np.array_equal(out["1"], v[0].reshape(-1, 4))
    # i (w + x i + y j + z k) = -x + w i - z j + y k, and so on
    assert np.array_equal(out["i"], np.stack([-x, w, -z, y], axis=1))
    assert np.array_equal(out["j"], np.stack([-y, z, w, -x], axis=1))
    assert np.array_equal(out["k"], np.stack([-z, -y, x, w], axis=1))


def test_fast_hurwitz_exact_norm_and_round_trip():
    d = 64
    g = np.random.default_rng(1)
    ql = (0.5 * g.choice([-1.0, 1.0], size=(d // 4, 4))).astype(np.float32)
    t = table_from_left(ql)
    x = g.integers(-64, 64, size=(20, d)).astype(np.float32)
    y = oracle.rotate_f32(x, oracle.ROT_QUAT_FAST, 0, t)
    ref = np.concatenate([x[:, 4 * j:4 * j + 4].astype(np.float64) @ left_matrix(ql[j]).T
                          for j in range(d // 4)], axis=1)
    assert np.array_equal(y.astype(np.float64), ref)  # halves of small integers: exact
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=0, atol=0)
    quat = workloads.random_quaternions(3, d)
    xd = g.standard_normal((5, d))
    back = oracle.unrotate_f64(oracle.rotate_f64(xd, oracle.ROT_QUAT_FAST, 0, quat),
                               oracle.ROT_QUAT_FAST, 0, quat)
    assert np.allclose(back, xd, rtol=0, atol=1e-12)


@pytest.mark.parametrize("b", [16, 64, 128])
def test_signed_hadamard_against_the_matrix(b):
    d = 128
    g = np.random.default_rng(b)
    x = g.integers(-100, 100, size=(8, d)).astype(np.float32)
    ones = np.ones(d, np.float32)
    assert np.array_equal(oracle.rotate_f32(x, oracle.ROT_HADAMARD_SIGNED, b, ones),
                          oracle.rotate_f32(x, oracle.ROT_HADAMARD, b))
    signs = workloads.random_signs(5, d)
    assert set(np.unique(signs)) == {-1.0, 1.0}
    Hm = np.array([[1]])
    while Hm.shape[0] < b:
        Hm = np.block([[Hm, Hm], [Hm, -Hm]])
    y = oracle.rotate_f32(x, oracle.ROT_HADAMARD_SIGNED, b, signs)
    cb = np.float64(oracle.hadamard_scale(b))
    xs = (x * signs).astype(np.int64)
    for t in range(0, d, b):
        # integer butterflies are exact; then one binary32 multiply by c_b
        ref = (xs[:, t:t + b] @ Hm.T).astype(np.float64)
        assert np.array_equal(y[:, t:t + b].astype(np.float64),
                              (ref.astype(np.float32) * np.float32(cb)).astype(np.float64))
    xd = g.standard_normal((4, d))
    back = oracle.unrotate_f64(oracle.rotate_f64(xd, oracle.ROT_HADAMARD_SIGNED, b, signs),
                               oracle.ROT_HADAMARD_SIGNED, b, signs)
    assert np.allclose(back, xd, rtol=0, atol=1e-12)


# --- IsoQuant-Full as one 4x4 matrix per block ------------------------------
# Pinned against the two multiplication matrices written out from the
# quaternion unit table (i^2 = j^2 = k^2 = ijk = -1), exact Hurwitz cases,
# the identity table, the two-product form to a few binary32 ulps, and
# orthogonality.

UNIT_PRODUCT = {  # (row unit) * (column unit) = sign, unit
    (0, 0): (1, 0), (0, 1): (1, 1), (0, 2): (1, 2), (0, 3): (1, 3),
    (1, 0): (1, 1), (1, 1): (-1, 0), (1, 2): (1, 3), (1, 3): (-1, 2),
    (2, 0): (1, 2), (2, 1): (-1, 3), (2, 2): (-1, 0), (2, 3): (1, 1),
    (3, 0): (1, 3), (3, 1): (1, 2), (3, 2): (-1, 1), (3, 3): (-1, 0),
}


def qmul(a, b):
    """Quaternion product from the unit multiplication table (float64)."""
    out = np.zeros(4)
    for i in range(4):
        for j in range(4):
            sg, u = UNIT_PRODUCT[(i, j)]
            out[u] += sg * a[i] * b[j]
    return out


def full_map_matrix(q8):
    """Columns: T(e_c) = qL e_c conj(qR) in float64."""
    qL = q8[:4].astype(np.float64)
    qRc = np.array([q8[4], -q8[5], -q8[6], -q8[7]], np.float64)
    return np.stack([qmul(qmul(qL, e), qRc) for e in np.eye(4)], axis=1)


def test_matrix_entries_against_the_unit_table():
    quat = workloads.random_quaternions(11, 128)
    for j in range(32):
        M = oracle.quat_matrix(quat[j])
        ref = full_map_matrix(quat[j].reshape(8))
        # four binary32 multiply-adds of terms at most 1 in size
        assert np.max(np.abs(M.astype(np.float64) - ref)) <= 4 * 2.0 ** -24


def test_matrix_hurwitz_exact_and_identity():
    g = np.random.default_rng(4)
    q = (0.5 * g.choice([-1.0, 1.0], size=(16, 8))).astype(np.float32)
    for j in range(16):
        assert np.array_equal(oracle.quat_matrix(q[j]).astype(np.float64), full_map_matrix(q[j]))
    ident = np.tile(np.array([1, 0, 0, 0, 1, 0, 0, 0], np.float32), (16, 1))
    assert np.array_equal(oracle.quat_matrix(ident[0]), np.eye(4, dtype=np.float32))
    x = g.standard_normal((6, 64)).astype(np.float32)
    assert np.array_equal(oracle.rotate_f32(x, oracle.ROT_QUAT_MAT, 0, ident.reshape(16, 2, 4)), x)
    # Hurwitz table on small integers: every product and sum is exact
    xi = g.integers(-50, 50, size=(6, 64)).astype(np.float32)
    y = oracle.rotate_f32(xi, oracle.ROT_QUAT_MAT, 0, q.reshape(16, 2, 4))
    ref = np.concatenate([xi[:, 4 * j:4 * j + 4].astype(np.float64) @ full_map_matrix(q[j]).T
                          for j in range(16)], axis=1)
    assert np.array_equal(y.astype(np.float64), ref)


def test_matrix_form_close_to_two_products_and_orthogonal():
    d = 128
    g = np.random.default_rng(6)
    quat = workloads.random_quaternions(2, d)
    x = g.standard_normal((50, d)).astype(np.float32)
    ym = oracle.rotate_f32(x, oracle.ROT_QUAT_MAT, 0, quat)
    yq = oracle.rotate_f32(x, oracle.ROT_QUAT, 0, quat)
    scale = np.abs(x).reshape(50, d // 4, 4).max(axis=2).repeat(4, axis=1)
    assert np.all(np.abs(ym - yq) <= 16 * 2.0 ** -24 * scale)
    assert np.any(ym != yq)  # a different rounding, not the same arithmetic
    for j in range(d // 4):
        M = oracle.quat_matrix(quat[j]).astype(np.float64)
        assert np.allclose(M @ M.T, np.eye(4), rtol=0, atol=1e-6)
    # the double-precision map is the binary32 matrix applied exactly; its
    # transpose undoes it to the matrix's distance from orthogonality
    xd = g.standard_normal((4, d))
    fwd = oracle.rotate_f64(xd, oracle.ROT_QUAT_MAT, 0, quat)
    for j in range(d // 4):
        M = oracle.quat_matrix(quat[j]).astype(np.float64)
        assert np.allclose(fwd[:, 4 * j:4 * j + 4], xd[:, 4 * j:4 * j + 4] @ M.T, rtol=0, atol=1e-13)
    back = oracle.unrotate_f64(fwd, oracle.ROT_QUAT_MAT, 0, quat)
    assert np.allclose(back, xd, rtol=0, atol=1e-5)
