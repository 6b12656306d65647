"""GPU parity of kvq_paged_decode_attn against the oracle's double-precision
attention over the same INT4 pages: max |out - oracle| <= 2e-3 (the target
stated for this method), over the five workloads' shapes (sampled sequences
at the full sizes) and the edge cases."""

import math

import numpy as np
import pytest
import torch

from bit_rotated_kv_block_b200 import kvq, workloads
from gpu_helpers import Pair, fill_workload, fused_step_vs_oracle

pytestmark = pytest.mark.gpu

TOL = 2e-3


def check(p, q, lens, L, table, sm):
    out, e = p.gpu_attention(q, lens, L, table, sm)
    ref, oe = p.oracle_attention(q, lens, L, table, sm)
    assert e == oe
    err = np.max(np.abs(out - ref)) if out.size else 0.0
    assert err <= TOL, f"max abs error {err}"
    return err


def test_tiny():
    w = workloads.tiny()
    p, _ = fill_workload(w)
    q = w.queries()
    check(p, q, w.seq_lens, 256, w.block_table, 1 / math.sqrt(w.d))


def test_llama8b_full_step():
    # 32 sequences x 4096 cached tokens, one appended token each, then decode
    w = workloads.llama8b()
    p, _ = fill_workload(w)
    k, v, ts, tp = w.step_tokens(0)
    e, oe = p.append(k, v, ts, tp, w.block_table)
    assert e == 0 and oe == 0
    p.assert_pools_equal()
    lens = w.seq_lens + 1
    check(p, w.queries(), lens, int(lens.max()), w.block_table, 1 / math.sqrt(w.d))


@pytest.mark.parametrize("rot", [workloads.ROT_HADAMARD, workloads.ROT_NONE])
def test_long70b_full(rot):
    # the full 8 x 32768 cache (pools checked bit-exact); every sequence and
    # query head of the one decode launch against the oracle
    w = workloads.long70b(rot_kind=rot)
    p, _ = fill_workload(w)
    p.assert_pools_equal()
    check(p, w.queries(), w.seq_lens, int(w.seq_lens.max()), w.block_table,
          1 / math.sqrt(w.d))


def test_long70b_full_fused_step():
    # 8 x 32767 cached tokens, then one fused step writes token 32768 of every
    # sequence (the last slot of its last page) and attends over 32768
    w = workloads.long70b(ctx=32767)
    p, _ = fill_workload(w)
    k_new, v_new, _, _ = w.step_tokens(0)
    lens = (w.seq_lens + 1).astype(np.int32)
    assert int(lens.max()) == 32768
    out, ref, e, oe = fused_step_vs_oracle(p, k_new, v_new, lens, w.block_table, w.queries(),
                                           1 / math.sqrt(w.d))
    assert e == 0 and oe == 0
    p.assert_pools_equal()
    assert np.max(np.abs(out - ref)) <= TOL


@pytest.mark.parametrize("rot", [workloads.ROT_HADAMARD, workloads.ROT_QUAT])
def test_ragged256_subset(rot):
    w = workloads.ragged256(rot_kind=rot)
    seqs = list(range(0, 128, 16))
    p, _ = fill_workload(w, seqs=seqs)
    # attend over the filled sequences only: a sub-table and their lengths
    table = w.block_table[seqs]
    lens = w.seq_lens[seqs]
    q = w.queries()[seqs]
    check(p, q, lens, int(w.seq_lens.max()), table, 1 / math.sqrt(w.d))


@pytest.mark.parametrize("d,H,G,P,rot,b", [(128, 2, 1, 16, 1, 128), (128, 2, 2, 32, 1, 64),
                                           (128, 1, 3, 16, 0, 0), (128, 2, 8, 64, 1, 16),
                                           (128, 3, 5, 16, 2, 0), (256, 2, 4, 16, 1, 256),
                                           (256, 1, 2, 32, 2, 0), (256, 2, 4, 64, 1, 32)])
def test_shapes_and_ragged_lengths(d, H, G, P, rot, b):
    g = np.random.default_rng(d * 7 + H + G + P + rot)
    lens = np.array([0, 1, 17, P, 3 * P + 5, 700], np.int32)
    S = len(lens)
    bt_stride = int(-(-lens.max() // P)) + 1
    NP = S * bt_stride + 3
    table = g.permutation(NP)[:S * bt_stride].reshape(S, bt_stride).astype(np.int32)
    quat = workloads.random_quaternions(2, d) if rot == 2 else None
    p = Pair(d, H, P, NP, rot, b, quat)
    ts = np.concatenate([np.full(n, s, np.int32) for s, n in enumerate(lens)])
    tp = np.concatenate([np.arange(n, dtype=np.int32) for n in lens])
    k = (g.standard_normal((len(ts), H, d)) * 2).astype(np.float16)
    v = (g.standard_normal((len(ts), H, d)) * 2).astype(np.float16)
    k[:, :, 5] *= 20
    e, oe = p.append(k, v, ts, tp, table)
    assert e == 0 and oe == 0
    q = g.standard_normal((S, H * G, d)).astype(np.float16)
    check(p, q, lens, int(lens.max()), table, 1 / math.sqrt(d))
    out, _ = p.gpu_attention(q, lens, int(lens.max()), table, 1 / math.sqrt(d))
    assert np.all(out[0] == 0)  # empty sequence


def test_peaked_attention_sink():
    # one very large key aligned with the query: softmax nearly one-hot
    g = np.random.default_rng(5)
    d, H, G, P = 128, 1, 4, 16
    L = 300
    table = np.arange(20, dtype=np.int32)[None]
    p = Pair(d, H, P, 20, 1, 128)
    k = g.standard_normal((L, H, d)).astype(np.float16)
    v = (g.standard_normal((L, H, d)) * 5).astype(np.float16)
    q = g.standard_normal((1, G, d)).astype(np.float16)
    k[7, 0] = (q[0, 0].astype(np.float32) * 3).astype(np.float16)
    e, _ = p.append(k, v, np.zeros(L, np.int32), np.arange(L, dtype=np.int32), table)
    assert e == 0
    check(p, q, np.array([L]), L, table, 1 / math.sqrt(d))


def test_invalid_page_and_length_flags():
    g = np.random.default_rng(9)
    d, H, G, P = 128, 2, 4, 16
    table = np.array([[0, 1, 2], [3, 4, 5]], np.int32)
    p = Pair(d, H, P, 6, 1, 128)
    lens = np.array([40, 40], np.int32)
    ts = np.repeat(np.arange(2, dtype=np.int32), 40)
    tp = np.tile(np.arange(40, dtype=np.int32), 2)
    k = g.standard_normal((80, H, d)).astype(np.float16)
    e, _ = p.append(k, k, ts, tp, table)
    assert e == 0
    bad = table.copy()
    bad[1, 1] = 77          # middle page of sequence 1 out of the pool
    q = g.standard_normal((2, H * G, d)).astype(np.float16)
    err = check(p, q, lens, 40, bad, 0.1)
    assert err <= TOL
    out, e = p.gpu_attention(q, lens, 40, bad, 0.1)
    assert e == kvq.ERRF_PAGE
    out, e = p.gpu_attention(q, np.array([40, 41], np.int32), 40, table, 0.1)
    assert e == kvq.ERRF_LEN and np.all(out[1] == 0)


def test_workspace_too_small_is_rejected():
    p = Pair(128, 2, 16, 4, 1, 128)
    q = torch.zeros((1, 8, 128), dtype=torch.float16, device="cuda")
    lens = torch.tensor([10], dtype=torch.int32, device="cuda")
    bt = torch.zeros((1, 4), dtype=torch.int32, device="cuda")
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(kvq.KvqError) as ei:
        kvq.paged_decode_attn(p.gpu, q, lens, 10, bt, p.kc, p.kp, p.vc, p.vp, workspace=ws)
    assert ei.value.status == 4
