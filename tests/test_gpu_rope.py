"""GPU parity of the optional rotary position embedding in front of the
rotation (a kvq_cache_desc with a RoPE table): key rows turned at their own
positions before rotation and quantization, bit-exact against the oracle in
the bulk and the small-batch append kernels and in the fused decode step;
the decode query turned at position seq_len - 1, attention within 2e-3 of
the oracle; positions past the table flagged."""

import math

import numpy as np
import pytest
import torch

import oracle
from bit_rotated_kv_block_b200 import kvq, workloads
from gpu_helpers import dev, fused_step_vs_oracle

pytestmark = pytest.mark.gpu

TOL = 2e-3


class RopePair:
    def __init__(self, d, H, P, NP, rot, b, quat, rope):
        self.gpu = kvq.Cache(d, H, P, NP, rot, b, quat, rope=rope)
        self.orc = oracle.Cache(d, H, P, NP, rot, b, quat, rope=rope)
        self.kc, self.kp = self.gpu.new_pools(fill=0xAA)
        self.vc, self.vp = self.gpu.new_pools(fill=0xAA)
        self.okc, self.okp = self.orc.alloc_pools(0xAA)
        self.ovc, self.ovp = self.orc.alloc_pools(0xAA)
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def append(self, k, v, ts, tp, table):
        self.err.zero_()
        kvq.quantize_append(self.gpu, dev(k), dev(v), dev(ts), dev(tp), dev(table), self.kc,
                            self.kp, self.vc, self.vp, err=self.err)
        oe = oracle.quantize_append(self.orc, k.view(np.uint16), v.view(np.uint16), ts, tp, table,
                                    self.okc, self.okp, self.ovc, self.ovp)
        torch.cuda.synchronize()
        return int(self.err.item()), oe

    def assert_pools_equal(self):
        assert np.array_equal(self.kc.cpu().numpy(), self.okc)
        assert np.array_equal(self.vc.cpu().numpy(), self.ovc)
        assert np.array_equal(self.kp.cpu().numpy().view(np.uint16).reshape(self.okp.shape), self.okp)
        assert np.array_equal(self.vp.cpu().numpy().view(np.uint16).reshape(self.ovp.shape), self.ovp)

    # gpu_helpers.fused_step_vs_oracle reads these names
    def okp_pool(self):
        return self.okp

    def oracle_attention(self, q, lens, L, table, sm):
        return oracle.paged_decode_attn(self.orc, q.view(np.uint16), lens, L, table,
                                        float(np.float32(sm)), self.okc, self.okp, self.ovc,
                                        self.ovp)


def make(rot, d=128, S=6, ctx=700, H=8, P=16):
    w = workloads.llama8b(S=S, ctx=ctx, spare_pages=8)
    b = {workloads.ROT_HADAMARD: 64, workloads.ROT_NONE: 0, workloads.ROT_QUAT: 0}[rot]
    quat = workloads.random_quaternions(3, d) if rot == workloads.ROT_QUAT else None
    rope = workloads.rope_table(4096, d)
    p = RopePair(d, H, P, w.NP, rot, b, quat, rope)
    return w, p


@pytest.mark.parametrize("rot", [workloads.ROT_HADAMARD, workloads.ROT_QUAT, workloads.ROT_NONE])
def test_append_with_rope_bit_exact(rot):
    # S x 700 tokens x 8 heads x {K, V} > 8192 rows: the bulk kernel; then one
    # token per sequence: the small-batch kernel
    w, p = make(rot)
    k, v, ts, tp = w.prefill_tokens()
    assert len(ts) * w.H * 2 > 8192
    e, oe = p.append(k, v, ts, tp, w.block_table)
    assert e == 0 and oe == 0
    p.assert_pools_equal()
    k1, v1, ts1, tp1 = w.step_tokens(0)
    e, oe = p.append(k1, v1, ts1, tp1, w.block_table)
    assert e == 0 and oe == 0
    p.assert_pools_equal()


@pytest.mark.parametrize("rot", [workloads.ROT_HADAMARD, workloads.ROT_QUAT])
def test_decode_and_fused_step_with_rope(rot):
    w, p = make(rot)
    k, v, ts, tp = w.prefill_tokens()
    assert p.append(k, v, ts, tp, w.block_table) == (0, 0)
    sm = 1 / math.sqrt(w.d)
    q = w.queries()
    p.err.zero_()
    out = kvq.paged_decode_attn(p.gpu, dev(q), dev(w.seq_lens), int(w.seq_lens.max()),
                                dev(w.block_table), p.kc, p.kp, p.vc, p.vp, sm_scale=sm,
                                err=p.err)
    ref, oe = p.oracle_attention(q, w.seq_lens, int(w.seq_lens.max()), w.block_table, sm)
    assert int(p.err.item()) == 0 and oe == 0
    assert np.max(np.abs(out.cpu().numpy() - ref)) <= TOL
    # fused step: the new token's key turned at position seq_len and written,
    # the query at the same position
    k_new, v_new, _, _ = w.step_tokens(1)
    lens = (w.seq_lens + 1).astype(np.int32)
    out1, ref1, e, oe = fused_step_vs_oracle(p, k_new, v_new, lens, w.block_table, w.queries(1),
                                             sm)
    assert e == 0 and oe == 0
    p.assert_pools_equal()
    assert np.max(np.abs(out1 - ref1)) <= TOL


def test_positions_past_the_table_are_flagged():
    d, H, P = 128, 2, 16
    rope = workloads.rope_table(40, d)
    p = RopePair(d, H, P, 8, workloads.ROT_HADAMARD, 128, None, rope)
    table = np.arange(8, dtype=np.int32).reshape(2, 4)
    k = np.ones((2, H, d), np.float16)
    e, oe = p.append(k, k, np.array([0, 1], np.int32), np.array([39, 40], np.int32), table)
    assert e == kvq.ERRF_POS and oe == oracle.ERR_POS
    p.assert_pools_equal()  # position 40 untouched on both sides
    q = torch.ones((2, 2 * H, d), dtype=torch.float16, device="cuda")
    p.err.zero_()
    out = kvq.paged_decode_attn(p.gpu, q, dev(np.array([40, 41], np.int32)), 41, dev(table),
                                p.kc, p.kp, p.vc, p.vp, err=p.err)
    torch.cuda.synchronize()
    assert int(p.err.item()) & kvq.ERRF_LEN
    assert torch.all(out[1] == 0)
