"""Pins the oracle's optional rotary position embedding (RoPE) in front of the
block rotation: adjacent channel pairs (2i, 2i+1) turned by the (cos, sin)
row of the token's position, in binary32 with every product and the
difference / sum rounded separately; keys at their own positions in the
append, the query at position seq_len - 1 in attention.

Pins: the identity at position 0; quarter turns that compose exactly
(products with 0 and +-1 are exact); binary32 agreement with complex
multiplication in float64 to two roundings; norm preservation; the attention
output against scaled_dot_product_attention with the query turned
independently; and the stored keys against independently turned keys within
the quantization bound.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from bit_rotated_kv_block_b200 import workloads


def quarter_turn_table(d):
    """Positions 0..3 turn every pair by 0, 90, 180 and 270 degrees."""
    cs = np.array([[1, 0], [0, 1], [-1, 0], [0, -1]], np.float32)
    return np.repeat(cs[:, None, :], d // 2, axis=1)


def complex_rope(x, cs):
    """x float64 [..][d], cs [..][d/2][2]: (x_2i + i x_2i+1) (c + i s)."""
    z = x[..., 0::2] + 1j * x[..., 1::2]
    w = cs[..., 0].astype(np.float64) + 1j * cs[..., 1].astype(np.float64)
    y = z * w
    out = np.empty_like(x)
    out[..., 0::2] = y.real
    out[..., 1::2] = y.imag
    return out


def test_identity_at_position_zero():
    x = np.random.default_rng(0).standard_normal((5, 64)).astype(np.float32)
    tbl = workloads.rope_table(4, 64)
    assert np.all(tbl[0, :, 0] == 1) and np.all(tbl[0, :, 1] == 0)
    y = oracle.rope_rows_f32(x, np.repeat(tbl[:1], 5, axis=0))
    assert np.array_equal(y, x)


def test_quarter_turns_compose_exactly():
    d = 32
    x = np.random.default_rng(1).standard_normal((1, d)).astype(np.float32)
    t = quarter_turn_table(d)
    one = oracle.rope_rows_f32(x, t[1:2])
    assert np.array_equal(one[0, 0::2], -x[0, 1::2]) and np.array_equal(one[0, 1::2], x[0, 0::2])
    assert np.array_equal(oracle.rope_rows_f32(one, t[1:2]), oracle.rope_rows_f32(x, t[2:3]))
    assert np.array_equal(oracle.rope_rows_f32(x, t[2:3]), -x)
    assert np.array_equal(oracle.rope_rows_f32(oracle.rope_rows_f32(x, t[2:3]), t[1:2]),
                          oracle.rope_rows_f32(x, t[3:4]))


def test_matches_complex_multiplication_and_keeps_the_norm():
    d, n = 128, 200
    g = np.random.default_rng(2)
    x = (g.standard_normal((n, d)) * 4).astype(np.float32)
    tbl = workloads.rope_table(4096, d)
    pos = g.integers(0, 4096, size=n)
    y = oracle.rope_rows_f32(x, tbl[pos])
    ref = complex_rope(x.astype(np.float64), tbl[pos])
    # each output: two rounded products and one rounded sum
    bound = 3 * 2.0 ** -24 * (np.abs(x[:, 0::2]) + np.abs(x[:, 1::2]))
    assert np.all(np.abs(y[:, 0::2] - ref[:, 0::2]) <= bound)
    assert np.all(np.abs(y[:, 1::2] - ref[:, 1::2]) <= bound)
    nx = np.linalg.norm(x.astype(np.float64), axis=1)
    assert np.allclose(np.linalg.norm(y.astype(np.float64), axis=1), nx, rtol=1e-6)


@pytest.mark.parametrize("rot,b", [(oracle.ROT_HADAMARD, 64), (oracle.ROT_NONE, 0)])
def test_append_and_attention_with_rope(rot, b):
    d, H, G, P = 64, 2, 2, 16
    lens = [40, 70]
    S = len(lens)
    g = np.random.default_rng(3)
    bt_stride = 6
    NP = S * bt_stride
    table = g.permutation(NP).reshape(S, bt_stride).astype(np.int32)
    rope = workloads.rope_table(128, d)
    cache = oracle.Cache(d, H, P, NP, rot, b, rope=rope)
    kc, kp = cache.alloc_pools(0)
    vc, vp = cache.alloc_pools(0)
    ts = np.concatenate([np.full(n, s, np.int32) for s, n in enumerate(lens)])
    tp = np.concatenate([np.arange(n, dtype=np.int32) for n in lens])
    k = (g.standard_normal((len(ts), H, d)) * 2).astype(np.float16)
    v = (g.standard_normal((len(ts), H, d)) * 3).astype(np.float16)
    assert oracle.quantize_append(cache, k.view(np.uint16), v.view(np.uint16), ts, tp, table,
                                  kc, kp, vc, vp) == 0
    # stored keys: R^-1 of the dequantized row is the key turned at its own
    # position, within the quantization error (|e_i| <= s16/2 in the rotated
    # basis, an orthogonal R keeps the Euclidean norm of the error)
    for t in range(len(ts)):
        s, j = ts[t], tp[t]
        page, slot = table[s, j // P], j % P
        xh = oracle.dequantize_rows(kc[page, :, slot], kp[page, :, slot, 0], kp[page, :, slot, 1])
        back = oracle.unrotate_f64(xh, rot, b)
        want = complex_rope(k[t].astype(np.float64), rope[j][None])
        s16 = oracle.half_bits_to_double(kp[page, :, slot, 0])
        err = np.linalg.norm(back - want, axis=1)
        assert np.all(err <= s16 / 2 * math.sqrt(d) * (1 + 1e-6) + 1e-5)
    # attention: the query turned at seq_len - 1, then sdpa over the dense rows
    q = g.standard_normal((S, H * G, d)).astype(np.float16)
    sm = 1 / math.sqrt(d)
    out, err = oracle.paged_decode_attn(cache, q.view(np.uint16), lens, max(lens), table, sm,
                                        kc, kp, vc, vp)
    assert err == 0
    for s, L in enumerate(lens):
        qt = complex_rope(q[s].astype(np.float64), np.repeat(rope[L - 1][None], H * G, axis=0))
        qhat = oracle.rotate_f64(qt, rot, b)
        K = np.zeros((H, L, d))
        V = np.zeros((H, L, d))
        for j in range(L):
            page, slot = table[s, j // P], j % P
            K[:, j] = oracle.dequantize_rows(kc[page, :, slot], kp[page, :, slot, 0],
                                             kp[page, :, slot, 1])
            V[:, j] = oracle.dequantize_rows(vc[page, :, slot], vp[page, :, slot, 0],
                                             vp[page, :, slot, 1])
        o = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qhat[:, None, :]), torch.from_numpy(np.repeat(K, G, axis=0)),
            torch.from_numpy(np.repeat(V, G, axis=0)), scale=sm)[:, 0].numpy()
        ref = oracle.unrotate_f64(o, rot, b)
        assert np.max(np.abs(out[s] - ref)) < 1e-12


def test_positions_outside_the_table_are_flagged():
    d, H, P = 64, 1, 16
    rope = workloads.rope_table(20, d)
    cache = oracle.Cache(d, H, P, 4, oracle.ROT_HADAMARD, 64, rope=rope)
    kc, kp = cache.alloc_pools(0xAA)
    vc, vp = cache.alloc_pools(0xAA)
    k = np.ones((2, H, d), np.float16)
    table = np.array([[0, 1, 2]], np.int32)
    e = oracle.quantize_append(cache, k.view(np.uint16), k.view(np.uint16),
                               np.array([0, 0], np.int32), np.array([19, 20], np.int32), table,
                               kc, kp, vc, vp)
    assert e == oracle.ERR_POS
    assert np.all(kc[1, 0, 4] == 0xAA)  # position 20 (page 1, slot 4) untouched
    q = np.ones((1, 1, d), np.float16)
    out, e = oracle.paged_decode_attn(cache, q.view(np.uint16), [21], 21, table, 0.1, kc, kp, vc, vp)
    assert e == oracle.ERR_LEN and np.all(out == 0)
