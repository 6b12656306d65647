"""GPU parity of kvq_quantize_append against the CPU oracle: packed codes,
binary16 scale/minimum and page placement bit-exact, untouched pool bytes
intact, over the workloads' shapes (tiny, Llama-3-8B prefill, every prefill
block size at full layer size, ragged head_dim 256 with Hadamard and
quaternion rotations) and the edge cases."""

import numpy as np
import pytest
import torch

import oracle
from bit_rotated_kv_block_b200 import kvq, workloads
from conftest import read_golden
from gpu_helpers import Pair, dev, fill_workload

pytestmark = pytest.mark.gpu


def test_tiny_bit_exact():
    w = workloads.tiny()
    p, _ = fill_workload(w)
    p.assert_pools_equal()


@pytest.mark.parametrize("b", [16, 32, 64, 128, 0])
def test_prefill_layer_full_size_every_block(b):
    # 65536 tokens x 8 heads x {K, V} of one layer, page 16, shuffled table
    w = workloads.prefill(rot_block=b)
    p, _ = fill_workload(w)
    p.assert_pools_equal()


def test_llama8b_prefill_full_size():
    w = workloads.llama8b()
    p, _ = fill_workload(w)
    p.assert_pools_equal()
    # then one decode-step token per sequence at position 4096
    k, v, ts, tp = w.step_tokens(0)
    e, oe = p.append(k, v, ts, tp, w.block_table)
    assert e == 0 and oe == 0
    p.assert_pools_equal()


@pytest.mark.parametrize("rot", [workloads.ROT_HADAMARD, workloads.ROT_QUAT])
def test_ragged_head_dim_256(rot):
    w = workloads.ragged256(rot_kind=rot)
    p, _ = fill_workload(w, seqs=range(0, 128, 9))
    p.assert_pools_equal()


def test_golden_rows_on_gpu():
    # the hand-worked rows of tests/golden/quant_rows_hand.txt, tiled to
    # head_dim 64 (tiling keeps the row minimum and maximum)
    g = read_golden("quant_rows_hand.txt")
    for row, kind, b in (("row1", kvq.ROT_NONE, 0), ("row2", kvq.ROT_HADAMARD, 16),
                         ("row3", kvq.ROT_NONE, 0), ("row4", kvq.ROT_HADAMARD, 16)):
        x = np.array([float(t) for t in g[row + "_x"].split()], np.float16)
        k = np.tile(x, 4).reshape(1, 1, 64)
        p = Pair(64, 1, 16, 2, kind, b)
        table = np.array([[1]], np.int32)
        e, _ = p.append(k, k, np.array([0]), np.array([3]), table, oracle_too=False)
        assert e == 0
        codes = p.kc[1, 0, 3].cpu().numpy()
        expect = np.array([int(t, 16) for t in g[row + "_packed"].split()], np.uint8)
        assert np.array_equal(codes, np.tile(expect, 4))
        word = int(p.kp[1, 0, 3].item()) & 0xFFFFFFFF
        assert word & 0xFFFF == int(g[row + "_s16"], 16)
        assert word >> 16 == int(g[row + "_m16"], 16)


@pytest.mark.parametrize("d,H,P,rot,b", [(128, 8, 16, 1, 128), (64, 3, 32, 1, 32),
                                         (256, 2, 64, 1, 256), (256, 4, 16, 2, 0),
                                         (128, 1, 16, 0, 0), (64, 5, 16, 2, 0)])
def test_ragged_token_batch_and_edges(d, H, P, rot, b):
    g = np.random.default_rng(d + H + P + rot)
    S, bt_stride = 5, 6
    NP = S * bt_stride + 7
    table = g.permutation(NP)[:S * bt_stride].reshape(S, bt_stride).astype(np.int32)
    T = 37
    token_seq = g.integers(0, S, size=T).astype(np.int32)
    token_seq[[4, 20]] = -1                                  # skipped tokens
    # distinct positions per sequence, straddling pages
    token_pos = np.zeros(T, np.int32)
    for s in range(S):
        idx = np.nonzero(token_seq == s)[0]
        token_pos[idx] = g.choice(bt_stride * P, size=len(idx), replace=False)
    quat = workloads.random_quaternions(7, d) if rot == 2 else None
    k = (g.standard_normal((T, H, d)) * g.uniform(0.01, 50, size=(T, H, 1))).astype(np.float16)
    v = (g.standard_normal((T, H, d)) * 3).astype(np.float16)
    # degenerate rows: constant, zero, negative zero, large, subnormal. The
    # large row stays inside the format's domain: every rotated value and
    # the scale fit binary16 (a quaternion block of +-30000 has norm 60000)
    k[0, 0] = 1.5
    k[1, 0] = 0.0
    v[1, 0] = -0.0
    k[2, 0, ::2] = 30000.0
    k[2, 0, 1::2] = -30000.0
    v[3, 0] = (g.standard_normal(d) * 1e-6).astype(np.float16)
    p = Pair(d, H, P, NP, rot, b, quat)
    e, oe = p.append(k, v, token_seq, token_pos, table)
    assert e == 0 and oe == 0
    p.assert_pools_equal()


@pytest.mark.parametrize("T,d,H,rot,b,qkv", [
    (520, 128, 8, 1, 64, False), (1201, 128, 8, 1, 128, False), (4999, 128, 8, 0, 0, False),
    (9000, 128, 8, 1, 32, False), (3000, 128, 8, 1, 16, False), (2000, 64, 8, 1, 64, False),
    (3001, 64, 3, 1, 32, False), (2500, 128, 5, 2, 0, False), (1700, 64, 4, 2, 0, False),
    (1200, 128, 8, 1, 128, True), (1200, 128, 8, 1, 64, True)])
def test_bulk_batches_ragged(T, d, H, rot, b, qkv):
    # batches above the warp-per-row path (T * H * 2 > 8192 rows): a few
    # work units per warp or CTA, a partial last unit, skipped tokens, an
    # odd head count, both channel ownerships of the streaming kernel
    # (b < d and b = d), quaternions, and rows read out of a fused
    # [T][(Hq + 2H) d] projection
    g = np.random.default_rng(T + d + H + b)
    P, S = 16, 3
    bt_stride = (T + P - 1) // P + 2
    NP = S * bt_stride + 5
    table = g.permutation(NP)[:S * bt_stride].reshape(S, bt_stride).astype(np.int32)
    token_seq = g.integers(0, S, size=T).astype(np.int32)
    token_seq[::97] = -1                                    # skipped tokens
    token_pos = np.zeros(T, np.int32)
    for s in range(S):
        idx = np.nonzero(token_seq == s)[0]
        token_pos[idx] = g.permutation(bt_stride * P)[:len(idx)]
    quat = workloads.random_quaternions(11, d) if rot == 2 else None
    k = (g.standard_normal((T, H, d)) * g.uniform(0.05, 20, size=(T, H, 1))).astype(np.float16)
    v = g.standard_normal((T, H, d)).astype(np.float16)
    k[1, 0] = 0.0                                           # degenerate rows
    v[2, 0] = 1.5
    p = Pair(d, H, P, NP, rot, b, quat)
    if not qkv:
        e, oe = p.append(k, v, token_seq, token_pos, table)
    else:
        Hq = 4 * H
        stride = (Hq + 2 * H) * d
        buf = g.standard_normal((T, stride)).astype(np.float16)
        buf[:, Hq * d:(Hq + H) * d] = k.reshape(T, H * d)
        buf[:, (Hq + H) * d:] = v.reshape(T, H * d)
        flat = buf.reshape(-1)
        bd = dev(buf).reshape(-1)
        e, oe = p.append(flat[Hq * d:], flat[(Hq + H) * d:], token_seq, token_pos, table,
                         tok_stride=stride, k_dev=bd[Hq * d:], v_dev=bd[(Hq + H) * d:])
    assert e == 0 and oe == 0
    p.assert_pools_equal()


def test_strided_input_from_fused_qkv():
    # K and V are slices of a [T][(Hq + 2H) * d] projection output
    g = np.random.default_rng(3)
    T, H, Hq, d, P = 50, 8, 32, 128, 16
    qkv = g.standard_normal((T, (Hq + 2 * H) * d)).astype(np.float16)
    stride = (Hq + 2 * H) * d
    flat = qkv.reshape(-1)
    k = flat[Hq * d:]
    v = flat[(Hq + H) * d:]
    table = g.permutation(8)[:4].reshape(1, 4).astype(np.int32)
    ts = np.zeros(T, np.int32)
    tp = np.arange(T, dtype=np.int32)
    p = Pair(d, H, P, 8, 1, 64)
    qkv_dev = dev(qkv).reshape(-1)
    e, oe = p.append(k, v, ts, tp, table, tok_stride=stride, k_dev=qkv_dev[Hq * d:],
                     v_dev=qkv_dev[(Hq + H) * d:])
    assert e == 0 and oe == 0
    p.assert_pools_equal()


def test_single_token_and_repeat_is_deterministic():
    w = workloads.tiny()
    k, v, ts, tp = w.prefill_tokens()
    p = Pair.for_workload(w)
    for _ in range(2):
        e, _ = p.append(k[:1], v[:1], ts[:1], tp[:1], w.block_table, oracle_too=False)
        assert e == 0
    e, oe = Pair.append(p, k[:1], v[:1], ts[:1], tp[:1], w.block_table)
    p.assert_pools_equal()


def test_invalid_entries_raise_flags_and_touch_nothing():
    d, H, P, NP = 128, 2, 16, 4
    table = np.array([[0, 1], [2, 99], [3, -4]], np.int32)
    g = np.random.default_rng(1)
    cases = [(5, 0, kvq.ERRF_SEQ), (0, 40, kvq.ERRF_POS), (0, -1, kvq.ERRF_POS),
             (1, 20, kvq.ERRF_PAGE), (2, 17, kvq.ERRF_PAGE)]
    for seq, pos, flag in cases:
        p = Pair(d, H, P, NP, 1, 128)
        k = g.standard_normal((1, H, d)).astype(np.float16)
        e, oe = p.append(k, k, np.array([seq]), np.array([pos]), table)
        assert e == flag and oe == flag
        p.assert_pools_equal()
        assert torch.all(p.kc == 0xAA) and torch.all(p.vc == 0xAA)
