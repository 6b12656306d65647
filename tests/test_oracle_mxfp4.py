"""Pins the oracle's microscaled FP4 cache format.

UltraQuant (page "UltraQuant: 4-bit KV caching for long agents", method
section): FP4 KV tensors with UE8M0 group scales and FP8 queries, taken by the
matrix cores' scaled multiply-accumulate. The reading is the Open Compute
Project microscaling (MX) element and scale formats: blocks of 32 channels, a
shared exponent X = floor(log2 amax) - emax stored as the byte X + 127, E2M1
(FP4) elements for K and V, E4M3 (FP8) elements for the query; round to
nearest, ties to even, saturating, sign kept.

Pinned against: the E2M1 value table written out from the format's bit
fields; hand-worked ties and saturation; brute-force nearest-value search on
dense grids (ties to the even mantissa); torch's own float8_e4m3fn cast (a
library conversion) for the query elements; the shared-exponent rule's
closed form (the scaled block maximum lands in [4, 8) for E2M1); attention
against torch's scaled_dot_product_attention in float64 on the dequantized
rows with the quantized query.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from bit_rotated_kv_block_b200 import workloads

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def e2m1_from_bits(code):
    """Value of an E2M1 code from its fields: sign, 2 exponent bits (bias 1),
    1 mantissa bit; exponent 0 is subnormal (m * 0.5)."""
    s, e, m = code >> 3, (code >> 1) & 3, code & 1
    v = m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
    return -v if s else v


def test_e2m1_table():
    for code in range(16):
        assert oracle.e2m1_value(code) == e2m1_from_bits(code)
    assert [e2m1_from_bits(c) for c in range(8)] == E2M1


def test_e2m1_hand_ties_saturation_and_sign():
    # midpoints go to the even mantissa: 0.25 -> 0, 0.75 -> 1, 1.25 -> 1,
    # 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4; above 6 saturates at 6
    cases = {0.0: 0, 0.25: 0, 0.26: 1, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6,
             5.01: 7, 6.0: 7, 6.9: 7, 7.0: 7, 1e9: 7, 0.5: 1, 1.5: 3, 3.0: 5}
    for t, code in cases.items():
        assert oracle.e2m1_encode(t) == code, t
        assert oracle.e2m1_encode(-t) == 8 | code, -t  # sign kept, -0 included


def test_e2m1_brute_force_nearest():
    grid = np.concatenate([np.linspace(-7.5, 7.5, 6001), [0.25 * k for k in range(-30, 31)]])
    for t in grid:
        code = oracle.e2m1_encode(float(t))
        v = oracle.e2m1_value(code)
        a = min(abs(t), 6.0)
        dists = [abs(a - g) for g in E2M1]
        best = min(dists)
        assert abs(abs(v) - a) == best
        ties = [i for i, dd in enumerate(dists) if dd == best]
        if len(ties) > 1:
            assert (code & 1) == 0  # even mantissa
        assert (code >> 3) == (1 if np.signbit(t) else 0)


def e4m3_torch_bits(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_against_torch_cast_and_table():
    g = np.random.default_rng(3)
    x = np.concatenate([g.standard_normal(4000) * 50, g.uniform(-448, 448, 2000),
                        g.standard_normal(2000) * 0.01, np.ldexp(np.arange(-12, 9.0), 0),
                        [0.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11, 448.0, -448.0, 440.0, 464.0 - 1e-3]])
    x = x.astype(np.float32)
    x = x[np.abs(x) <= 448]
    ours = np.array([oracle.e4m3_encode(float(v)) for v in x], np.uint8)
    ref = e4m3_torch_bits(x)
    # torch's cast of a negative value that rounds to zero gives -0 too
    assert np.array_equal(ours, ref)
    for code in range(256):
        if code & 0x7F == 0x7F:
            continue  # NaN encodings
        v = oracle.e4m3_value(code)
        assert oracle.e4m3_encode(v) == code or (v == 0.0 and code in (0, 0x80))
    assert oracle.e4m3_value(0x7E) == 448.0 and oracle.e4m3_value(0x01) == 2.0 ** -9
    assert oracle.e4m3_value(0x08) == 2.0 ** -6 and oracle.e4m3_value(0x38) == 1.0
    assert oracle.e4m3_encode(1000.0) == 0x7E  # saturating


def test_shared_exponent_rule():
    for k in range(-20, 20):
        for f in (1.0, 1.3, 1.999):
            amax = np.float32(f * 2.0 ** k)
            assert oracle.mx_exponent(float(amax), 2) == k - 2
            assert oracle.mx_exponent(float(amax), 8) == k - 8
            assert 4.0 <= float(amax) / 2.0 ** (k - 2) < 8.0
    assert oracle.mx_exponent(0.0, 2) == -127


def test_row_hand_worked():
    # one block: amax 7 -> X = 2 - 2 = 0 (scale byte 127), elements as above
    y = np.zeros(32, np.float32)
    vals = [0.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0, -0.1, -2.6]
    y[:len(vals)] = vals
    codes, scales = oracle.mxfp4_quantize_rows(y[None])
    assert scales[0, 0] == 127
    expect = [0, 0, 2, 2, 4, 4, 6, 6, 7, 7, 8, 8 | 5] + [0] * (32 - len(vals))
    got = [(codes[0, k // 2] >> (4 * (k % 2))) & 15 for k in range(32)]
    assert got == expect
    # all-zero block: exponent byte 0, codes 0
    codes, scales = oracle.mxfp4_quantize_rows(np.zeros((1, 64), np.float32))
    assert np.all(scales == 0) and np.all(codes == 0)


def test_row_brute_force_and_bound():
    g = np.random.default_rng(9)
    y = (g.standard_normal((40, 128)) * np.exp(g.uniform(-4, 4, (40, 1)))).astype(np.float32)
    y[3, 5] = 1e-30  # a tiny value in an otherwise normal block
    codes, scales = oracle.mxfp4_quantize_rows(y)
    for r in range(40):
        for i in range(128):
            X = int(scales[r, i // 32]) - 127
            c = (codes[r, i // 2] >> (4 * (i % 2))) & 15
            t = float(y[r, i]) / 2.0 ** X
            amax = float(np.max(np.abs(y[r, 32 * (i // 32):32 * (i // 32) + 32])))
            assert X == math.floor(math.log2(amax)) - 2
            a = min(abs(t), 6.0)
            best = min(abs(a - v) for v in E2M1)
            assert abs(abs(e2m1_from_bits(c)) - a) == best
            # error bound: half the grid step of the element's binade
            # (0.25 below 2, 0.5 in [2, 4), 1 in [4, 6]), or the saturation
            # overshoot above 6
            err = abs(e2m1_from_bits(c) * 2.0 ** X - float(y[r, i]))
            half = 0.25 if a < 2 else (0.5 if a < 4 else 1.0)
            assert err <= max(half, abs(t) - 6.0) * 2.0 ** X


def test_query_values_against_torch():
    g = np.random.default_rng(4)
    y = (g.standard_normal((20, 128)) * 3).astype(np.float32)
    out = oracle.mxfp8_values(y)
    for r in range(20):
        for b in range(4):
            blk = y[r, 32 * b:32 * b + 32]
            X = math.floor(math.log2(float(np.max(np.abs(blk))))) - 8
            t = (blk.astype(np.float64) / 2.0 ** X).astype(np.float32)
            # the block maximum lands in [256, 512): above 448 the MX rule
            # saturates, where torch's cast (no saturation) gives NaN
            t = np.clip(t, -448, 448)
            ref = torch.tensor(t).to(torch.float8_e4m3fn).to(torch.float64).numpy() * 2.0 ** X
            assert np.array_equal(out[r, 32 * b:32 * b + 32], ref)


def build_fp4(rot, b, d, H, P, lens, seed, quat=None):
    g = np.random.default_rng(seed)
    S = len(lens)
    bt_stride = max((int(n) + P - 1) // P for n in lens) + 1
    NP = S * bt_stride + 2
    table = g.permutation(NP)[:S * bt_stride].reshape(S, bt_stride).astype(np.int32)
    cache = oracle.Cache(d, H, P, NP, rot, b, quat, fmt=oracle.FMT_MXFP4)
    kc, kp = cache.alloc_pools(0xAA)
    vc, vp = cache.alloc_pools(0xAA)
    ts = np.concatenate([np.full(n, s, np.int32) for s, n in enumerate(lens)])
    tp = np.concatenate([np.arange(n, dtype=np.int32) for n in lens])
    k = (g.standard_normal((len(ts), H, d)) * 2).astype(np.float16)
    k[:, :, 3] *= 12
    v = (g.standard_normal((len(ts), H, d)) * 3).astype(np.float16)
    assert oracle.quantize_append(cache, k.view(np.uint16), v.view(np.uint16), ts, tp, table,
                                  kc, kp, vc, vp) == 0
    return cache, table, k, v, ts, tp, (kc, kp, vc, vp)


@pytest.mark.parametrize("rot,b", [(oracle.ROT_HADAMARD, 64), (oracle.ROT_NONE, 0),
                                   (oracle.ROT_QUAT, 0)])
def test_append_places_rows_of_the_row_quantizer(rot, b):
    d, H, P = 128, 2, 16
    quat = workloads.random_quaternions(1, d) if rot == oracle.ROT_QUAT else None
    cache, table, k, v, ts, tp, (kc, kp, vc, vp) = build_fp4(rot, b, d, H, P, [37, 20], 5, quat)
    touched = np.zeros(kc.shape[:3], bool)
    for t in range(len(ts)):
        page, slot = table[ts[t], tp[t] // P], tp[t] % P
        touched[page, :, slot] = True
        for src, codes, params in ((k, kc, kp), (v, vc, vp)):
            y = oracle.rotate_f32(src[t].astype(np.float32), rot, b, quat)
            c, s = oracle.mxfp4_quantize_rows(y)
            assert np.array_equal(codes[page, :, slot], c)
            assert np.array_equal(params[page, :, slot], s)
    # untouched slots keep their sentinel bytes
    assert np.all(kc[~touched] == 0xAA) and np.all(vp[~touched] == 0xAA)


@pytest.mark.parametrize("rot,b", [(oracle.ROT_HADAMARD, 128), (oracle.ROT_QUAT, 0)])
def test_attention_against_sdpa(rot, b):
    d, H, P, G = 128, 2, 16, 4
    lens = [45, 1, 70]
    quat = workloads.random_quaternions(2, d) if rot == oracle.ROT_QUAT else None
    cache, table, k, v, ts, tp, pools = build_fp4(rot, b, d, H, P, lens, 8, quat)
    g = np.random.default_rng(11)
    S, Hq = len(lens), H * G
    q = (g.standard_normal((S, Hq, d))).astype(np.float16)
    sm = 1 / math.sqrt(d)
    out, err = oracle.paged_decode_attn(cache, q.view(np.uint16), lens, max(lens), table, sm,
                                        *pools)
    assert err == 0
    kx, _ = oracle.dequantize_pages(cache, lens, max(lens), table, pools[0], pools[1], False)
    vx, _ = oracle.dequantize_pages(cache, lens, max(lens), table, pools[2], pools[3], False)
    # dequantized rows in double (the float32 export is exact for these values)
    for s in range(S):
        L = lens[s]
        for hq in range(Hq):
            h = hq // G
            y = oracle.rotate_f32(q[s, hq].astype(np.float32), rot, b, quat)
            qq = oracle.mxfp8_values(y)
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.tensor(qq)[None, None, None], torch.tensor(kx[s, :L, h].astype(np.float64))[None, None],
                torch.tensor(vx[s, :L, h].astype(np.float64))[None, None], scale=sm)[0, 0, 0].numpy()
            ref = oracle.unrotate_f64(ref, rot, b, quat)
            assert np.allclose(out[s, hq], ref, rtol=0, atol=1e-12)


def test_dequantize_export_values():
    d, H, P = 128, 1, 16
    cache, table, k, v, ts, tp, (kc, kp, vc, vp) = build_fp4(oracle.ROT_NONE, 0, d, H, P, [30], 3)
    x, err = oracle.dequantize_pages(cache, [30], 30, table, kc, kp, False)
    assert err == 0
    for j in range(30):
        page, slot = table[0, j // P], j % P
        for i in range(d):
            c = (kc[page, 0, slot, i // 2] >> (4 * (i % 2))) & 15
            X = int(kp[page, 0, slot, i // 32]) - 127
            assert x[0, j, 0, i] == e2m1_from_bits(c) * 2.0 ** X
