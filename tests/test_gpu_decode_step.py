"""GPU parity of the fused decode step kvq_decode_step: the new token of every
sequence is written exactly as kvq_quantize_append writes it (pools bit-exact
against the oracle and against the two-call path) and the attention over the
updated cache is within 2e-3 of the oracle and equal to the two-call path."""

import math

import numpy as np
import pytest
import torch

from bit_rotated_kv_block_b200 import kvq, workloads
from gpu_helpers import Pair, dev, fill_workload, fused_step_vs_oracle

pytestmark = pytest.mark.gpu

TOL = 2e-3


def step_both_ways(w, p, k_new, v_new, lens, table, q):
    """Fused step on p's pools; the two-call path on copies; the oracle on p's
    oracle pools. Returns (fused out, two-call out, oracle out, flags)."""
    L = int(lens.max())
    sm = 1 / math.sqrt(w.d)
    kc2, kp2, vc2, vp2 = p.kc.clone(), p.kp.clone(), p.vc.clone(), p.vp.clone()
    err2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    ts = np.arange(w.S, dtype=np.int32)
    tp = (lens - 1).astype(np.int32)
    keep = lens >= 1
    ts_dev = dev(np.where(keep, ts, -1).astype(np.int32))
    kvq.quantize_append(p.gpu, dev(k_new), dev(v_new), ts_dev, dev(np.maximum(tp, 0)), dev(table),
                        kc2, kp2, vc2, vp2, err=err2)
    out2 = kvq.paged_decode_attn(p.gpu, dev(q), dev(lens), L, dev(table), kc2, kp2, vc2, vp2,
                                 sm_scale=sm, err=err2)
    p.err.zero_()
    out1 = kvq.decode_step(p.gpu, dev(q), dev(k_new), dev(v_new), dev(lens), L, dev(table), p.kc,
                           p.kp, p.vc, p.vp, sm_scale=sm, err=p.err)
    torch.cuda.synchronize()
    # oracle: the same append, then attention
    import oracle
    oe = oracle.quantize_append(p.orc, k_new.view(np.uint16), v_new.view(np.uint16),
                                np.where(keep, ts, -1).astype(np.int32),
                                np.maximum(tp, 0).astype(np.int32), table, p.okc,
                                p.okp.reshape(p.orc.NP, p.orc.H, p.orc.P, 2), p.ovc, p.ovp)
    ref, oe2 = p.oracle_attention(q, lens, L, table, sm)
    # the two GPU paths leave identical pools and outputs
    for a, b in ((p.kc, kc2), (p.kp, kp2), (p.vc, vc2), (p.vp, vp2)):
        assert torch.equal(a, b)
    o1, o2 = out1.cpu().numpy(), out2.cpu().numpy()
    assert np.array_equal(o1, o2)
    assert int(p.err.item()) == int(err2.item()) == (oe | oe2)
    return o1.astype(np.float64), ref


def test_llama8b_step():
    w = workloads.llama8b(S=6, ctx=1000, spare_pages=8)
    p, _ = fill_workload(w)
    k_new, v_new, _, _ = w.step_tokens(0)
    lens = (w.seq_lens + 1).astype(np.int32)
    out, ref = step_both_ways(w, p, k_new, v_new, lens, w.block_table, w.queries())
    p.assert_pools_equal()
    assert np.max(np.abs(out - ref)) <= TOL


@pytest.mark.parametrize("rot", [workloads.ROT_HADAMARD, workloads.ROT_QUAT, workloads.ROT_NONE])
def test_ragged_head_dim_256_step(rot):
    # lengths chosen so that new tokens open a fresh page, end one, or are the
    # only token of their sequence
    w = workloads.ragged256(S=5, lo=40, hi=200, rot_kind=rot)
    w.seq_lens = np.array([32, 47, 0, 150, 63], np.int32)
    pages = [(int(n) + 1 + w.P - 1) // w.P for n in w.seq_lens]
    w.NP = sum(pages) + 3
    perm = np.random.default_rng(5).permutation(w.NP).astype(np.int32)
    w.block_table = np.full((w.S, max(pages)), -1, np.int32)
    off = 0
    for s_, n in enumerate(pages):
        w.block_table[s_, :n] = perm[off:off + n]
        off += n
    p, _ = fill_workload(w)
    k_new, v_new, _, _ = w.step_tokens(1)
    lens = (w.seq_lens + 1).astype(np.int32)
    out, ref = step_both_ways(w, p, k_new, v_new, lens, w.block_table, w.queries(1))
    p.assert_pools_equal()
    assert np.max(np.abs(out - ref)) <= TOL


def test_long70b_shaped_step_gqa8():
    w = workloads.long70b(S=2, ctx=2000)
    p, _ = fill_workload(w)
    k_new, v_new, _, _ = w.step_tokens(0)
    lens = (w.seq_lens + 1).astype(np.int32)
    out, ref = step_both_ways(w, p, k_new, v_new, lens, w.block_table, w.queries())
    p.assert_pools_equal()
    assert np.max(np.abs(out - ref)) <= TOL


def test_new_token_page_outside_pool_is_flagged():
    w = workloads.llama8b(S=3, ctx=160, spare_pages=4)
    p, _ = fill_workload(w)
    k_new, v_new, _, _ = w.step_tokens(0)
    lens = (w.seq_lens + 1).astype(np.int32)
    table = w.block_table.copy()
    table[1, 160 // w.P] = w.NP + 3  # the page of sequence 1's new token
    p.err.zero_()
    kvq.decode_step(p.gpu, dev(w.queries()), dev(k_new), dev(v_new), dev(lens), int(lens.max()),
                    dev(table), p.kc, p.kp, p.vc, p.vp, err=p.err)
    torch.cuda.synchronize()
    assert int(p.err.item()) & kvq.ERRF_PAGE


def test_llama8b_full_size_step_matches_two_calls_and_oracle():
    # the bench's workload and launch configuration: 32 sequences x 4096
    # cached tokens, one new token each; the fused step and the two-call path
    # leave identical pools and outputs, and both equal the oracle's
    w = workloads.llama8b()
    p, _ = fill_workload(w)
    k_new, v_new, ts, tp = w.step_tokens(0)
    lens = (w.seq_lens + 1).astype(np.int32)
    L = int(lens.max())
    q = dev(w.queries())
    kc2, kp2, vc2, vp2 = p.kc.clone(), p.kp.clone(), p.vc.clone(), p.vp.clone()
    bt = dev(w.block_table)
    kvq.quantize_append(p.gpu, dev(k_new), dev(v_new), dev(ts), dev(tp), bt, kc2, kp2, vc2, vp2)
    out2 = kvq.paged_decode_attn(p.gpu, q, dev(lens), L, bt, kc2, kp2, vc2, vp2)
    out1, ref, e, oe = fused_step_vs_oracle(p, k_new, v_new, lens, w.block_table, w.queries(),
                                            1 / math.sqrt(w.d))
    assert e == 0 and oe == 0
    for a, b in ((p.kc, kc2), (p.kp, kp2), (p.vc, vc2), (p.vp, vp2)):
        assert torch.equal(a, b)
    assert np.array_equal(out1, out2.cpu().numpy().astype(np.float64))
    p.assert_pools_equal()
    assert np.max(np.abs(out1 - ref)) <= TOL
