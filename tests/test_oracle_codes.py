"""Pins the oracle's 2- and 3-bit integer formats and the 16-entry table
format, and the offline table calibration.

* INT2 / INT3 (IsoQuant page, Abstract: bit widths {2, 3, 4}): the INT4 rule
  with Q = 2^bits - 1 levels above zero; codes packed little-endian into a
  bit stream. Pinned by hand-packed bytes, brute-force pack/unpack, hand rows
  (an exact ramp, a tie row), the nearest-level property and the error bound.
* LUT4 (UltraQuant page, method section: a calibrated 16-entry table in place
  of the uniform levels): the INT4 statistics, the code of the nearest table
  level with ties to the lower index. Pinned by brute-force nearest search,
  the identity table (INT4's codes except at exact ties), and attention
  against torch's scaled_dot_product_attention on the dequantized rows.
* Calibration: the result is a Lloyd-Max fixed point on its samples (every
  level within half a grid step of its cell's mean, cells by nearest level)
  and quantizes those samples with a smaller error than the uniform levels.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from bit_rotated_kv_block_b200 import calibrate, workloads


def test_packing_by_hand():
    # INT2: codes (1, 2, 3, 0) -> 1 | 2 << 2 | 3 << 4 = 0x39
    y = np.array([[0, 1, 2, 3] * 4], np.float32)  # ramp: m 0, s 1
    c, s16, m16 = oracle.quantize_rows_fmt(y, oracle.FMT_INT2)
    assert oracle.half_bits_to_double(s16)[0] == 1.0 and c[0, 0] == 0 | 1 << 2 | 2 << 4 | 3 << 6
    # INT3: codes 0..7 -> the 24-bit value sum(i << 3i) in three bytes
    y = np.array([list(range(8)) * 2], np.float32)
    c, s16, _ = oracle.quantize_rows_fmt(y, oracle.FMT_INT3)
    v = sum(i << (3 * i) for i in range(8))
    assert list(c[0, :3]) == [v & 0xFF, (v >> 8) & 0xFF, v >> 16]
    assert oracle.half_bits_to_double(s16)[0] == 1.0


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_pack_unpack_brute_force(bits):
    g = np.random.default_rng(bits)
    d = 64
    c = g.integers(0, 1 << bits, size=(50, d)).astype(np.int32)
    # pack by the definition (bit stream, little-endian) here, unpack in the oracle
    packed = np.zeros((50, d * bits // 8), np.uint8)
    for r in range(50):
        acc = 0
        for i in range(d):
            acc |= int(c[r, i]) << (i * bits)
        packed[r] = np.frombuffer(acc.to_bytes(d * bits // 8, "little"), np.uint8)
    assert np.array_equal(oracle.unpack_codes_bits(packed, d, bits), c)


@pytest.mark.parametrize("fmt,Q", [(oracle.FMT_INT2, 3), (oracle.FMT_INT3, 7)])
def test_integer_rows_nearest_and_bound(fmt, Q):
    g = np.random.default_rng(Q)
    bits = {3: 2, 7: 3}[Q]
    y = (g.standard_normal((60, 64)) * np.exp(g.uniform(-3, 3, (60, 1)))).astype(np.float32)
    y[0] = 1.25  # constant row: scale 0, all codes 0
    codes, s16, m16 = oracle.quantize_rows_fmt(y, fmt)
    c = oracle.unpack_codes_bits(codes, 64, bits)
    s = oracle.half_bits_to_double(s16)[:, None]
    m = oracle.half_bits_to_double(m16)[:, None]
    assert np.all(c[0] == 0) and s[0, 0] == 0
    assert np.all(c >= 0) and np.all(c <= Q)
    rows = s[:, 0] > 0
    # every value lies in [m, m + Q s]; its code is a nearest level
    yd = y.astype(np.float64)
    assert np.all(yd[rows] >= m[rows]) and np.all(yd[rows] <= m[rows] + Q * s[rows])
    err = np.abs(c * s + m - yd)
    assert np.all(err[rows] <= s[rows] * (0.5 + 64 * 2.0 ** -24))
    # argmin -> 0, argmax -> Q
    assert np.all(c[rows, np.argmin(y[rows], axis=1)] == 0)
    assert np.all(c[rows, np.argmax(y[rows], axis=1)] == Q)


def test_integer_tie_row_by_hand():
    # INT2, row (0, 0.5, 1.5, 2.5, 3) repeated: m 0, s 1, u = the values;
    # ties to even: 0.5 -> 0, 1.5 -> 2, 2.5 -> 2
    y = np.array([[0, 0.5, 1.5, 2.5, 3, 3, 3, 3] * 2], np.float32)
    codes, s16, _ = oracle.quantize_rows_fmt(y, oracle.FMT_INT2)
    assert oracle.half_bits_to_double(s16)[0] == 1.0
    c = oracle.unpack_codes_bits(codes, 16, 2)[0]
    assert list(c[:5]) == [0, 0, 2, 2, 3]


def lut_levels(seed=0):
    """16 strictly increasing levels on the 1/16 grid in [0.25, 14.5]."""
    g = np.random.default_rng(seed)
    grid = np.arange(5, 232) / 16.0  # 0.3125 .. 14.4375
    t = np.sort(g.choice(grid, size=14, replace=False))
    return np.concatenate([[0.25], t, [14.5]]).astype(np.float32)


def test_lut_brute_force_nearest_lower_tie():
    t = lut_levels()
    g = np.random.default_rng(5)
    y = (g.standard_normal((40, 64)) * 2).astype(np.float32)
    codes, s16, m16 = oracle.quantize_rows_fmt(y, oracle.FMT_LUT4, t)
    c = oracle.unpack_codes_bits(codes, 64, 4)
    s = np.float32(oracle.half_bits_to_double(s16)).astype(np.float32)
    m = np.float32(oracle.half_bits_to_double(m16)).astype(np.float32)
    for r in range(40):
        inv = np.float32(1.0) / s[r]
        u = (y[r] - m[r]).astype(np.float64) * np.float64(inv)  # exact product
        d = np.abs(u[:, None] - t.astype(np.float64)[None, :])
        best = d.min(axis=1)
        lowest = np.argmax(d == best[:, None], axis=1)  # the lower index on ties
        assert np.array_equal(c[r], lowest)


def test_lut_identity_table_matches_int4_off_ties():
    t = np.arange(16, dtype=np.float32)
    g = np.random.default_rng(6)
    y = (g.standard_normal((30, 64)) * 3).astype(np.float32)
    cl, sl, ml = oracle.quantize_rows_fmt(y, oracle.FMT_LUT4, t)
    ci, si, mi = oracle.quantize_rows(y)
    assert np.array_equal(sl, si) and np.array_equal(ml, mi)
    a = oracle.unpack_codes_bits(cl, 64, 4)
    b = oracle.unpack_codes_bits(ci, 64, 4)
    diff = a != b
    # where they differ, INT4 rounded an exact half up to an even code and
    # the table took the lower level
    assert np.all(b[diff] - a[diff] == 1) and np.all(b[diff] % 2 == 0)
    # a hand tie: u = 0.5 exactly -> LUT 0, INT4 0 (even); u = 1.5 -> LUT 1, INT4 2
    y = np.array([[0, 0.5, 1.5, 15] * 16], np.float32)
    cl, _, _ = oracle.quantize_rows_fmt(y, oracle.FMT_LUT4, t)
    assert list(oracle.unpack_codes_bits(cl, 64, 4)[0, :4]) == [0, 0, 1, 15]


@pytest.mark.parametrize("fmt", [oracle.FMT_INT2, oracle.FMT_INT3, oracle.FMT_LUT4])
def test_append_and_attention_against_sdpa(fmt):
    d, H, P, G = 64, 2, 16, 2
    lens = [37, 1, 50]
    g = np.random.default_rng(12)
    S = len(lens)
    bt_stride = 4
    NP = S * bt_stride + 2
    table = g.permutation(NP)[:S * bt_stride].reshape(S, bt_stride).astype(np.int32)
    lv = lut_levels(3) if fmt == oracle.FMT_LUT4 else None
    cache = oracle.Cache(d, H, P, NP, oracle.ROT_HADAMARD, 32, fmt=fmt, levels=lv)
    kc, kp = cache.alloc_pools(0xAA)
    vc, vp = cache.alloc_pools(0xAA)
    ts = np.concatenate([np.full(n, s, np.int32) for s, n in enumerate(lens)])
    tp = np.concatenate([np.arange(n, dtype=np.int32) for n in lens])
    k = (g.standard_normal((len(ts), H, d)) * 2).astype(np.float16)
    v = (g.standard_normal((len(ts), H, d)) * 3).astype(np.float16)
    assert oracle.quantize_append(cache, k.view(np.uint16), v.view(np.uint16), ts, tp, table,
                                  kc, kp, vc, vp) == 0
    # the placed rows are the row quantizer's
    bits = {oracle.FMT_INT2: 2, oracle.FMT_INT3: 3}.get(fmt, 4)
    for t in range(len(ts)):
        page, slot = table[ts[t], tp[t] // P], tp[t] % P
        yk = oracle.rotate_f32(k[t].astype(np.float32), oracle.ROT_HADAMARD, 32)
        c, s16, m16 = oracle.quantize_rows_fmt(yk, fmt, lv)
        assert np.array_equal(kc[page, :, slot], c)
        assert np.array_equal(kp[page, :, slot, 0], s16) and np.array_equal(kp[page, :, slot, 1], m16)
    q = g.standard_normal((S, H * G, d)).astype(np.float16)
    sm = 1 / math.sqrt(d)
    out, err = oracle.paged_decode_attn(cache, q.view(np.uint16), lens, max(lens), table, sm,
                                        kc, kp, vc, vp)
    assert err == 0
    kx, _ = oracle.dequantize_pages(cache, lens, max(lens), table, kc, kp, False)
    vx, _ = oracle.dequantize_pages(cache, lens, max(lens), table, vc, vp, False)
    for s in range(S):
        L = lens[s]
        qh = oracle.rotate_f64(q[s].astype(np.float64), oracle.ROT_HADAMARD, 32)
        for hq in range(H * G):
            h = hq // G
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.tensor(qh[hq])[None, None, None],
                torch.tensor(kx[s, :L, h].astype(np.float64))[None, None],
                torch.tensor(vx[s, :L, h].astype(np.float64))[None, None], scale=sm)[0, 0, 0]
            ref = oracle.unrotate_f64(ref.numpy(), oracle.ROT_HADAMARD, 32)
            assert np.allclose(out[s, hq], ref, rtol=0, atol=1e-9)
    # dequantized values: level (or code) times s16 plus m16, exactly
    page, slot = table[0, 0], 0
    c = oracle.unpack_codes_bits(kc[page, 0, slot], d, bits)
    s = oracle.half_bits_to_double(kp[page, 0, slot, 0])
    m = oracle.half_bits_to_double(kp[page, 0, slot, 1])
    vals = lv.astype(np.float64)[c] if fmt == oracle.FMT_LUT4 else c.astype(np.float64)
    assert np.array_equal(kx[0, 0, 0].astype(np.float64), (vals * s + m).astype(np.float32))


def test_calibration_is_a_lloyd_max_fixed_point_and_beats_uniform():
    w = workloads.prefill(rot_block=64)
    g = np.random.default_rng(7)
    rows = g.standard_normal((3000, 128)) * w.channel_mult[0][None, :] \
        if w.channel_mult is not None else g.standard_normal((3000, 128))
    t = calibrate.calibrate_levels(rows, 64)
    assert t.dtype == np.float32 and np.all(np.diff(t) > 0)
    assert np.all(t >= 0) and np.all(t <= 15) and np.all(t * 16 == np.round(t * 16))
    u = calibrate.normalised_codes_domain(calibrate.rotate_rows(rows, 64)).ravel()
    # nearest-level cells (ties to the lower) and their means
    mids = 0.5 * (t[1:].astype(np.float64) + t[:-1])
    cell = np.searchsorted(mids, u, side="left")
    for k in range(16):
        sel = u[cell == k]
        if len(sel) > 100:
            assert abs(sel.mean() - t[k]) <= 1 / 32 + 0.02, (k, sel.mean(), t[k])
    mse_t = np.mean((u - t[cell]) ** 2)
    mse_u = np.mean((u - np.clip(np.rint(u), 0, 15)) ** 2)
    assert mse_t < mse_u


def test_level_table_rounding_keeps_strictly_increasing_grid_levels():
    # the decode's integer path needs 16 t integral and strictly increasing
    # levels: crowded inputs move up one grid step, and down from the top
    # when the grid runs out
    lo = calibrate.round_to_grid(np.zeros(16))
    assert np.array_equal(lo * 16, np.arange(16))
    hi = calibrate.round_to_grid(np.full(16, 15.0))
    assert np.array_equal(hi * 16, np.arange(225, 241))
    g = np.random.default_rng(3)
    for _ in range(200):
        t = calibrate.round_to_grid(g.uniform(-2, 17, 16) ** g.choice([1, 2]) % 15.5)
        assert t.dtype == np.float32 and np.all(np.diff(t) > 0)
        assert np.all(t >= 0) and np.all(t <= 15) and np.all(t * 16 == np.round(t * 16))
    # Lloyd-Max on 16 separated clusters (symmetric about the integers 1..14,
    # point masses at 0 and 15) moves a perturbed start onto the cluster
    # means, the integers
    u = np.concatenate([k + np.linspace(-0.45, 0.45, 99) for k in range(1, 15)] +
                       [np.zeros(99), np.full(99, 15.0)])
    t = calibrate.lloyd_max(u, init=np.arange(16) + 0.04 * (-1.0) ** np.arange(16))
    assert np.max(np.abs(t - np.arange(16))) < 1e-9
