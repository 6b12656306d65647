"""Pins the oracle's decode attention and dense export.

Attention over the rotated INT4 cache ("SAW-INT4" Key takeaway: the cache
serves fused attention; the query is rotated by the same orthogonal R so that
q . k is preserved) is compared with torch's scaled_dot_product_attention in
float64 on the dequantized rows, with a pure-Python brute force on a tiny
case, and with the invariants: one cached token returns R^-1 vhat_0, equal
keys return the mean of the values, and attention over the rotated cache
equals plain attention over the un-rotated dequantized rows.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from bit_rotated_kv_block_b200 import workloads


def build_cache(rot, b, d, H, P, S, lens, seed, quat=None, same_keys=False):
    g = np.random.default_rng(seed)
    bt_stride = max((int(n) + P - 1) // P for n in lens) + 1
    NP = S * bt_stride + 3
    table = g.permutation(NP)[:S * bt_stride].reshape(S, bt_stride).astype(np.int32)
    cache = oracle.Cache(d, H, P, NP, rot, b, quat)
    kc, kp = cache.alloc_pools(0)
    vc, vp = cache.alloc_pools(0)
    token_seq = np.concatenate([np.full(n, s, np.int32) for s, n in enumerate(lens)])
    token_pos = np.concatenate([np.arange(n, dtype=np.int32) for n in lens])
    T = len(token_seq)
    k = (g.standard_normal((T, H, d)) * 2).astype(np.float16)
    if same_keys:
        k[:] = k[0]
    v = (g.standard_normal((T, H, d)) * 3).astype(np.float16)
    k[:, :, 1] *= 15  # an outlier channel
    assert oracle.quantize_append(cache, k.view(np.uint16), v.view(np.uint16), token_seq,
                                  token_pos, table, kc, kp, vc, vp) == 0
    return cache, table, (kc, kp, vc, vp)


def dense_rows(cache, table, lens, codes, params):
    """Exact dequantized (rotated) rows [S][Lmax][H][d] in float64."""
    S = len(lens)
    out = np.zeros((S, max(lens), cache.H, cache.d))
    for s in range(S):
        for j in range(lens[s]):
            page = table[s, j // cache.P]
            out[s, j] = oracle.dequantize_rows(codes[page, :, j % cache.P],
                                               params[page, :, j % cache.P, 0],
                                               params[page, :, j % cache.P, 1])
    return out


CASES = [(oracle.ROT_HADAMARD, 16, 16, 2, 2, 4), (oracle.ROT_HADAMARD, 32, 64, 2, 4, 4),
         (oracle.ROT_NONE, 0, 64, 2, 3, 4), (oracle.ROT_QUAT, 0, 64, 2, 4, 8)]


@pytest.mark.parametrize("rot,b,d,H,G,P", CASES)
def test_attention_matches_sdpa_float64(rot, b, d, H, G, P):
    lens = [1, 7, 37, 20]
    S = len(lens)
    quat = workloads.random_quaternions(4, d) if rot == oracle.ROT_QUAT else None
    cache, table, (kc, kp, vc, vp) = build_cache(rot, b, d, H, P, S, lens, 1, quat)
    Hq = H * G
    q = (np.random.default_rng(2).standard_normal((S, Hq, d))).astype(np.float16)
    sm = 1 / math.sqrt(d)
    out, err = oracle.paged_decode_attn(cache, q.view(np.uint16), lens, max(lens), table, sm,
                                        kc, kp, vc, vp)
    assert err == 0
    K = dense_rows(cache, table, lens, kc, kp)
    V = dense_rows(cache, table, lens, vc, vp)
    qhat = oracle.rotate_f64(q.astype(np.float64), rot, b, quat)
    for s in range(S):
        L = lens[s]
        kq = torch.from_numpy(np.repeat(K[s, :L].transpose(1, 0, 2), G, axis=0))   # [Hq][L][d]
        vq = torch.from_numpy(np.repeat(V[s, :L].transpose(1, 0, 2), G, axis=0))
        qq = torch.from_numpy(qhat[s][:, None, :])                                  # [Hq][1][d]
        o = torch.nn.functional.scaled_dot_product_attention(qq, kq, vq, scale=sm)
        ref = oracle.unrotate_f64(o[:, 0].numpy(), rot, b, quat)
        assert np.max(np.abs(out[s] - ref)) < 1e-12


def test_attention_brute_force_tiny():
    d, H, G, P = 16, 1, 2, 4
    lens = [5]
    cache, table, (kc, kp, vc, vp) = build_cache(oracle.ROT_HADAMARD, 16, d, H, P, 1, lens, 3)
    q = np.random.default_rng(4).standard_normal((1, G, d)).astype(np.float16)
    out, _ = oracle.paged_decode_attn(cache, q.view(np.uint16), lens, 5, table, 0.25, kc, kp, vc, vp)
    # explicit R = H_16 / 4 from the Sylvester recursion
    Hm = np.array([[1]])
    while Hm.shape[0] < 16:
        Hm = np.block([[Hm, Hm], [Hm, -Hm]])
    R = Hm / 4.0
    for g in range(G):
        qh = [sum(R[i][j] * float(q[0, g, j]) for j in range(d)) for i in range(d)]
        keys, vals = [], []
        for j in range(5):
            page, slot = table[0, j // P], j % P
            cs = [(int(kc[page, 0, slot, i // 2]) >> (4 * (i % 2))) & 15 for i in range(d)]
            cv = [(int(vc[page, 0, slot, i // 2]) >> (4 * (i % 2))) & 15 for i in range(d)]
            sk, mk = [float(oracle.half_bits_to_double(np.array([kp[page, 0, slot, t]]))[0]) for t in (0, 1)]
            sv, mv = [float(oracle.half_bits_to_double(np.array([vp[page, 0, slot, t]]))[0]) for t in (0, 1)]
            keys.append([c * sk + mk for c in cs])
            vals.append([c * sv + mv for c in cv])
        z = [0.25 * sum(a * b for a, b in zip(qh, kk)) for kk in keys]
        zm = max(z)
        w = [math.exp(t - zm) for t in z]
        tot = sum(w)
        ot = [sum(w[j] / tot * vals[j][i] for j in range(5)) for i in range(d)]
        o = [sum(R[i][j] * ot[j] for j in range(d)) for i in range(d)]
        assert np.max(np.abs(np.array(o) - out[0, g])) < 1e-12


def hurwitz_table(d, seed):
    """Quaternions with every component +-1/2: exactly unit in binary32."""
    g = np.random.default_rng(seed)
    return (0.5 * g.choice([-1.0, 1.0], size=(d // 4, 2, 4))).astype(np.float32)


@pytest.mark.parametrize("rot,b,qtable", [(oracle.ROT_HADAMARD, 32, None),
                                         (oracle.ROT_QUAT, 0, "hurwitz"),
                                         (oracle.ROT_QUAT, 0, "random")])
def test_attention_preserves_dot_products(rot, b, qtable):
    # attention over the rotated cache == plain attention over R^-1 khat, R^-1 vhat
    d, H, G, P = 64, 2, 2, 4
    lens = [9, 30]
    quat = None
    if qtable == "hurwitz":
        quat = hurwitz_table(d, 6)
    elif qtable == "random":
        quat = workloads.random_quaternions(6, d)
    cache, table, (kc, kp, vc, vp) = build_cache(rot, b, d, H, P, 2, lens, 5, quat)
    q = np.random.default_rng(6).standard_normal((2, H * G, d)).astype(np.float16)
    out, _ = oracle.paged_decode_attn(cache, q.view(np.uint16), lens, 30, table, 0.125,
                                      kc, kp, vc, vp)
    # a random table is unit only to binary32 rounding, so T scales dot
    # products by |qL|^2 |qR|^2 = 1 + O(1e-7): allow for that there; the
    # Hurwitz table is exactly unit and must meet the tight bound
    tol = 1e-5 if qtable == "random" else 1e-12
    K = oracle.unrotate_f64(dense_rows(cache, table, lens, kc, kp), rot, b, quat)
    V = oracle.unrotate_f64(dense_rows(cache, table, lens, vc, vp), rot, b, quat)
    for s, L in enumerate(lens):
        for g in range(H * G):
            h = g // G
            z = 0.125 * K[s, :L, h] @ q[s, g].astype(np.float64)
            p = np.exp(z - z.max())
            p /= p.sum()
            assert np.max(np.abs(p @ V[s, :L, h] - out[s, g])) < tol


def test_single_token_and_equal_keys():
    d, H, G, P, b = 64, 2, 2, 4, 64
    cache, table, (kc, kp, vc, vp) = build_cache(oracle.ROT_HADAMARD, b, d, H, P, 1, [1], 7)
    q = np.random.default_rng(8).standard_normal((1, H * G, d)).astype(np.float16)
    out, _ = oracle.paged_decode_attn(cache, q.view(np.uint16), [1], 1, table, 0.125, kc, kp, vc, vp)
    V = dense_rows(cache, table, [1], vc, vp)
    for g in range(H * G):
        assert np.max(np.abs(out[0, g] - oracle.unrotate_f64(V[0, 0, g // G], 1, b))) < 1e-12
    # equal keys -> uniform weights -> mean of the values
    cache, table, (kc, kp, vc, vp) = build_cache(oracle.ROT_HADAMARD, b, d, H, P, 1, [13], 9,
                                                 same_keys=True)
    out, _ = oracle.paged_decode_attn(cache, q.view(np.uint16), [13], 13, table, 0.125,
                                      kc, kp, vc, vp)
    V = dense_rows(cache, table, [13], vc, vp)
    for g in range(H * G):
        mean = oracle.unrotate_f64(V[0, :13, g // G].mean(axis=0), 1, b)
        assert np.max(np.abs(out[0, g] - mean)) < 1e-12


def test_attention_edge_cases_and_flags():
    d, H, G, P = 16, 1, 2, 4
    cache, table, (kc, kp, vc, vp) = build_cache(oracle.ROT_HADAMARD, 16, d, H, P, 2, [8, 8], 10)
    q = np.ones((3, G, d), np.float16).view(np.uint16)
    bt = np.zeros((3, table.shape[1]), np.int32)
    bt[:2] = table
    # seq 1: second page entry invalid -> its tokens are excluded, flag 1
    bt[1, 1] = cache.NP + 5
    out, err = oracle.paged_decode_attn(cache, q, [8, 8, 0], 8, bt, 0.25, kc, kp, vc, vp)
    assert err == oracle.ERR_PAGE
    assert np.all(out[2] == 0)  # empty sequence
    ref, _ = oracle.paged_decode_attn(cache, q[1:2], [4], 8, bt[1:2], 0.25, kc, kp, vc, vp)
    assert np.max(np.abs(out[1] - ref[0])) < 1e-14
    # invalid length -> flag 8 and zeros
    out, err = oracle.paged_decode_attn(cache, q[:1], [9], 8, bt[:1], 0.25, kc, kp, vc, vp)
    assert err == oracle.ERR_LEN and np.all(out == 0)


def test_fp16_baseline_attention_matches_sdpa():
    g = np.random.default_rng(12)
    d, H, G, P, NP = 32, 2, 4, 8, 11
    lens = [19, 40]
    table = g.permutation(NP)[:10].reshape(2, 5).astype(np.int32)
    k16 = g.standard_normal((NP, H, P, d)).astype(np.float16)
    v16 = g.standard_normal((NP, H, P, d)).astype(np.float16)
    q = g.standard_normal((2, H * G, d)).astype(np.float16)
    out, err = oracle.paged_decode_attn_fp16(d, H, P, NP, q.view(np.uint16), lens, 40, table,
                                             0.2, k16.view(np.uint16), v16.view(np.uint16))
    assert err == 0
    for s, L in enumerate(lens):
        K = np.stack([k16[table[s, j // P], :, j % P] for j in range(L)]).astype(np.float64)
        V = np.stack([v16[table[s, j // P], :, j % P] for j in range(L)]).astype(np.float64)
        kq = torch.from_numpy(np.repeat(K.transpose(1, 0, 2), G, axis=0))
        vq = torch.from_numpy(np.repeat(V.transpose(1, 0, 2), G, axis=0))
        qq = torch.from_numpy(q[s].astype(np.float64)[:, None, :])
        o = torch.nn.functional.scaled_dot_product_attention(qq, kq, vq, scale=0.2)[:, 0].numpy()
        assert np.max(np.abs(o - out[s])) < 1e-12


@pytest.mark.parametrize("unrotate,fp32", [(0, 1), (1, 1), (0, 0), (1, 0)])
def test_dequantize_pages(unrotate, fp32):
    d, H, P, b = 64, 2, 4, 32
    lens = [6, 11]
    cache, table, (kc, kp, vc, vp) = build_cache(oracle.ROT_HADAMARD, b, d, H, P, 2, lens, 13)
    sentinel = np.float32(-12345.0) if fp32 else np.uint16(0xABCD)
    out = np.full((2, 12, H, d), sentinel, np.float32 if fp32 else np.uint16)
    out, err = oracle.dequantize_pages(cache, lens, 12, table, kc, kp, unrotate, fp32, out)
    assert err == 0
    exact = dense_rows(cache, table, lens, kc, kp)
    for s, L in enumerate(lens):
        ref = exact[s, :L]
        if unrotate:
            ref = oracle.unrotate_f64(ref, 1, b)
        if fp32:
            if unrotate:
                assert np.max(np.abs(out[s, :L] - ref)) <= 1e-6 * np.max(np.abs(ref))
            else:
                assert np.array_equal(out[s, :L], ref.astype(np.float32))
        else:
            got = oracle.half_bits_to_double(out[s, :L])
            if unrotate:
                assert np.all(np.abs(got - ref) <= 2 ** -11 * np.abs(ref) + 2 ** -24)
            else:
                assert np.array_equal(out[s, :L], ref.astype(np.float16).view(np.uint16))
        assert np.all(out[s, L:] == sentinel)


def test_reconstruction_mse_shrinks_with_rotation_on_outliers():
    # property the method rests on (rotation spreads outlier channels): with
    # two x20 channels, Hadamard rows reconstruct with lower MSE than none
    w = workloads.tiny()
    k, _, _, _ = w.prefill_tokens()
    x = k.astype(np.float32).reshape(-1, w.d)
    mses = {}
    for b in (0, 16, 128):
        kind = oracle.ROT_HADAMARD if b else oracle.ROT_NONE
        y = oracle.rotate_f32(x, kind, b)
        c, s16, m16 = oracle.quantize_rows(y)
        xh = oracle.dequantize_rows(c, s16, m16)
        if b:
            xh = oracle.unrotate_f64(xh, kind, b)
        mses[b] = oracle.reconstruction_mse(k.view(np.uint16).reshape(-1, w.d), xh)
    assert mses[128] < mses[16] < mses[0]
