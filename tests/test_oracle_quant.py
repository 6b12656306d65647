"""Pins the oracle's token-wise INT4 quantizer, nibble packing and paged
placement ("SAW-INT4" Summary/Method: token-wise INT4 fused into paged
KV-cache layouts).

Pins: four hand-worked rows (golden fixture, worked in exact rationals), a
constant row, the nearest-level property by brute force over all 16 levels,
the range guarantee x in [m16, m16 + 15 s16], the error bound
|x - xhat| <= s16 (1/2 + 64 * 2^-24), argmin -> 0 and argmax -> 15, the
uniform-noise model MSE ~ E[s^2]/12, the nibble order, and brute-force
placement with sentinel-filled pools and the error flags.
"""

import numpy as np
import pytest

import oracle
from bit_rotated_kv_block_b200 import workloads
from conftest import read_golden


def _hex_bytes(s):
    return np.array([int(t, 16) for t in s.split()], np.uint8)


@pytest.mark.parametrize("row", ["row1", "row2", "row3", "row4"])
def test_hand_worked_rows(row):
    g = read_golden("quant_rows_hand.txt")
    x = np.array([float(t) for t in g[row + "_x"].split()], np.float32)
    # inputs are binary16 values
    assert np.array_equal(x.astype(np.float16).astype(np.float32), x)
    if g[row + "_rotation"] == "hadamard16":
        y = oracle.rotate_f32(x[None], oracle.ROT_HADAMARD, 16)
    else:
        y = x[None]
    codes, s16, m16 = oracle.quantize_rows(y)
    assert int(s16[0]) == int(g[row + "_s16"], 16)
    assert int(m16[0]) == int(g[row + "_m16"], 16)
    assert np.array_equal(oracle.unpack_codes(codes)[0],
                          np.array([int(t) for t in g[row + "_codes"].split()]))
    assert np.array_equal(codes[0], _hex_bytes(g[row + "_packed"]))


def test_identity_levels_row():
    # (0, 1, ..., 15) repeated: m16 = 0, s16 = 1, codes = values, zero error
    x = np.tile(np.arange(16, dtype=np.float32), 8)[None]
    codes, s16, m16 = oracle.quantize_rows(x)
    assert int(s16[0]) == 0x3C00 and int(m16[0]) == 0
    assert np.array_equal(oracle.unpack_codes(codes)[0], np.arange(128) % 16)
    assert np.array_equal(oracle.dequantize_rows(codes, s16, m16)[0], x[0].astype(np.float64))


@pytest.mark.parametrize("value", [0.0, -0.0, 3.25, -7.5, 2.0 ** -20])
def test_constant_row_binary16_value(value):
    # a constant binary16 value: m16 = value exactly, s16 = 0, all codes 0
    x = np.full((1, 128), value, np.float32)
    codes, s16, m16 = oracle.quantize_rows(x)
    assert int(s16[0]) == 0
    assert np.all(codes == 0)
    assert oracle.half_bits_to_double(m16)[0] == value
    if value == 0.0:
        assert int(m16[0]) == 0  # -0 normalised to +0


def test_constant_row_between_binary16_values():
    # 1e-3 is not a binary16 value: m16 rounds below it, the scale is the
    # gap over 15 levels rounded up (here to a few subnormal quanta, so the
    # shared code is not 15), and every element takes the same code
    x = np.full((1, 128), 1e-3, np.float32)
    codes, s16, m16 = oracle.quantize_rows(x)
    c = oracle.unpack_codes(codes)[0]
    assert np.all(c == c[0])
    xhat = oracle.dequantize_rows(codes, s16, m16)[0]
    s = oracle.half_bits_to_double(s16)[0]
    assert 0 < s and np.all(np.abs(xhat - np.float64(np.float32(1e-3))) <= s / 2)


def _rows(n, d, seed, outliers=True):
    g = np.random.default_rng(seed)
    x = g.standard_normal((n, d)).astype(np.float32)
    if outliers:
        x[:, 3] *= 20
        x[:, d // 2 + 13] *= 20
    scale = np.exp(g.uniform(np.log(1e-3), np.log(1e3), size=(n, 1))).astype(np.float32)
    x = (x * scale).astype(np.float16).astype(np.float32)
    return x


@pytest.mark.parametrize("d,rot,b", [(128, oracle.ROT_NONE, 0), (128, oracle.ROT_HADAMARD, 128),
                                     (128, oracle.ROT_HADAMARD, 16), (256, oracle.ROT_HADAMARD, 256),
                                     (256, oracle.ROT_QUAT, 0)])
def test_quantizer_bounds_and_nearest_level(d, rot, b):
    x = _rows(2000, d, d + b + rot)
    quat = workloads.random_quaternions(1, d) if rot == oracle.ROT_QUAT else None
    y = oracle.rotate_f32(x, rot, b, quat)
    codes, s16, m16 = oracle.quantize_rows(y)
    c = oracle.unpack_codes(codes)
    s = oracle.half_bits_to_double(s16)[:, None]
    m = oracle.half_bits_to_double(m16)[:, None]
    yd = y.astype(np.float64)
    # range guarantee from the directed roundings
    assert np.all(yd >= m)
    assert np.all(yd <= m + 15 * s)
    # error bound
    xhat = c * s + m
    assert np.all(np.abs(yd - xhat) <= s * (0.5 + 64 * 2 ** -24))
    # nearest level: no other level is closer by more than the rounding slack
    levels = np.arange(16)[None, None, :] * s[:, :, None] + m[:, :, None]
    dist = np.abs(yd[:, :, None] - levels)
    best = dist.min(axis=2)
    chosen = np.abs(yd - xhat)
    assert np.all(chosen <= best + s * 64 * 2 ** -24)
    # extremes map to the end codes when the row is not constant
    nz = s[:, 0] > 0
    am = np.argmin(yd, axis=1)
    ax = np.argmax(yd, axis=1)
    r = np.arange(len(y))
    assert np.all(c[r[nz], am[nz]] == 0)
    assert np.all(c[r[nz], ax[nz]] == 15)


def test_quantization_noise_matches_uniform_model():
    # rotated Gaussian rows: interior errors are ~ uniform on [-s/2, s/2]
    x = _rows(8192, 128, 99, outliers=False)
    y = oracle.rotate_f32(x, oracle.ROT_HADAMARD, 128)
    codes, s16, m16 = oracle.quantize_rows(y)
    xhat = oracle.dequantize_rows(codes, s16, m16)
    s = oracle.half_bits_to_double(s16)
    mse_rel = np.mean(((y - xhat) / s[:, None]) ** 2)
    assert abs(mse_rel - 1 / 12) / (1 / 12) < 0.05


def test_nibble_order():
    # codes 0..15 then 15..0: byte k = c[2k] | c[2k+1] << 4
    x = np.concatenate([np.arange(16), np.arange(15, -1, -1)]).astype(np.float32)
    x = np.tile(x, 4)[None]
    codes, s16, m16 = oracle.quantize_rows(x)
    assert int(s16[0]) == 0x3C00
    assert codes[0, 0] == 0x10 and codes[0, 1] == 0x32 and codes[0, 7] == 0xFE
    assert codes[0, 8] == 0xEF and codes[0, 15] == 0x01


def _small_cache(rot=oracle.ROT_HADAMARD, b=32, d=64, H=3, P=4, NP=11):
    quat = workloads.random_quaternions(3, d) if rot == oracle.ROT_QUAT else None
    return oracle.Cache(d, H, P, NP, rot, b, quat)


@pytest.mark.parametrize("rot,b", [(oracle.ROT_HADAMARD, 32), (oracle.ROT_NONE, 0),
                                   (oracle.ROT_QUAT, 0)])
def test_append_places_rows_and_keeps_sentinels(rot, b):
    cache = _small_cache(rot, b)
    S, bt_stride = 3, 3
    g = np.random.default_rng(5)
    table = g.permutation(cache.NP)[:S * bt_stride].reshape(S, bt_stride).astype(np.int32)
    # tokens: a ragged mix, positions straddling pages, one skipped (seq -1)
    token_seq = np.array([0, 0, 1, 2, 2, 2, 1, -1, 0], np.int32)
    token_pos = np.array([0, 5, 3, 4, 9, 11, 4, 2, 6], np.int32)
    T = len(token_seq)
    k = g.standard_normal((T, cache.H, cache.d)).astype(np.float16)
    v = g.standard_normal((T, cache.H, cache.d)).astype(np.float16)
    kc, kp = cache.alloc_pools(0xAA)
    vc, vp = cache.alloc_pools(0xAA)
    err = oracle.quantize_append(cache, k.view(np.uint16), v.view(np.uint16), token_seq,
                                 token_pos, table, kc, kp, vc, vp)
    assert err == 0
    touched = np.zeros((cache.NP, cache.H, cache.P), bool)
    for t in range(T):
        if token_seq[t] < 0:
            continue
        page = table[token_seq[t], token_pos[t] // cache.P]
        slot = token_pos[t] % cache.P
        for src, codes, params in ((k, kc, kp), (v, vc, vp)):
            y = oracle.rotate_f32(src[t].astype(np.float32), rot, b, cache.quat)
            c_ref, s_ref, m_ref = oracle.quantize_rows(y)
            assert np.array_equal(codes[page, :, slot], c_ref)
            assert np.array_equal(params[page, :, slot, 0], s_ref)
            assert np.array_equal(params[page, :, slot, 1], m_ref)
        touched[page, :, slot] = True
    # every (seq, pos) went to a distinct slot, nothing else was written
    assert touched.sum() == cache.H * int((token_seq >= 0).sum())
    for codes, params in ((kc, kp), (vc, vp)):
        assert np.all(codes[~touched] == 0xAA)
        assert np.all(params[~touched] == 0xAAAA)


def test_append_error_flags():
    cache = _small_cache()
    table = np.array([[0, 1, 2], [3, 99, -5]], np.int32)
    kc, kp = cache.alloc_pools(0xAA)
    vc, vp = cache.alloc_pools(0xAA)
    k = np.ones((1, cache.H, cache.d), np.float16).view(np.uint16)

    def run(seq, pos):
        return oracle.quantize_append(cache, k, k, np.array([seq], np.int32),
                                      np.array([pos], np.int32), table, kc, kp, vc, vp)

    assert run(2, 0) == oracle.ERR_SEQ
    assert run(0, 12) == oracle.ERR_POS       # 12 / 4 = 3 >= bt_stride
    assert run(0, -1) == oracle.ERR_POS
    assert run(1, 4) == oracle.ERR_PAGE       # entry 99 >= NP
    assert run(1, 8) == oracle.ERR_PAGE       # entry -5
    assert run(-1, 0) == 0                    # skipped silently
    assert np.all(kc == 0xAA) and np.all(vp == 0xAAAA)


def test_distinct_slots_brute_force():
    w = workloads.llama8b(S=4, ctx=300)
    seen = set()
    for s in range(w.S):
        for pos in range(int(w.seq_lens[s]) + 1):
            key = (int(w.block_table[s, pos // w.P]), pos % w.P)
            assert key not in seen
            seen.add(key)


def test_upward_binary32_sub_and_div_are_smallest_upper_bounds():
    # checked against exact rational arithmetic: r >= exact and the next
    # binary32 value below r is < exact (or r == exact)
    from fractions import Fraction
    g = np.random.default_rng(17)
    a = (g.standard_normal(3000) * np.exp(g.uniform(-20, 20, 3000))).astype(np.float32)
    b = (g.standard_normal(3000) * np.exp(g.uniform(-20, 20, 3000))).astype(np.float32)
    for x, y in zip(a, b):
        for r, exact in ((oracle.sub_ru(x, y), Fraction(float(x)) - Fraction(float(y))),
                         (oracle.div_ru(x, np.float32(15)), Fraction(float(x)) / 15)):
            fr = Fraction(float(r))
            below = Fraction(float(np.nextafter(r, np.float32(-np.inf))))
            assert fr >= exact and (fr == exact or below < exact)
