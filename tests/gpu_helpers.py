"""Shared set-up for the GPU parity tests: the same seeded inputs go to the
CUDA library (through the C ABI) and to the CPU oracle."""

import numpy as np
import torch

import oracle
from bit_rotated_kv_block_b200 import kvq


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


class Pair:
    """One paged cache built twice: GPU pools through libkvq, host pools through
    the oracle, both started from the same sentinel bytes."""

    def __init__(self, d, H, P, NP, rot_kind, rot_block=0, quat=None, fill=0xAA,
                 fmt=kvq.FMT_INT4, levels=None):
        self.fmt = fmt
        self.gpu = kvq.Cache(d, H, P, NP, rot_kind, rot_block, quat, fmt=fmt, levels=levels)
        self.orc = oracle.Cache(d, H, P, NP, rot_kind, rot_block, quat, fmt=fmt, levels=levels)
        self.kc, self.kp = self.gpu.new_pools(fill=fill)
        self.vc, self.vp = self.gpu.new_pools(fill=fill)
        self.okc, self.okp = self.orc.alloc_pools(fill)
        self.ovc, self.ovp = self.orc.alloc_pools(fill)
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")

    @classmethod
    def for_workload(cls, w, fill=0xAA, fmt=kvq.FMT_INT4, levels=None):
        return cls(w.d, w.H, w.P, w.NP, w.rot_kind, w.rot_block, w.quat, fill, fmt, levels)

    def okp_pool(self):
        """The oracle's K params pool as its append writes it."""
        if self.fmt == kvq.FMT_MXFP4:
            return self.okp
        return self.okp.reshape(self.orc.NP, self.orc.H, self.orc.P, 2)

    def append(self, k, v, token_seq, token_pos, block_table, oracle_too=True, tok_stride=None,
               k_dev=None, v_dev=None):
        """k, v: float16 numpy [T][H][d] (or wider rows with tok_stride)."""
        self.err.zero_()
        kd = dev(k) if k_dev is None else k_dev
        vd = dev(v) if v_dev is None else v_dev
        bt = dev(block_table.astype(np.int32))
        kvq.quantize_append(self.gpu, kd, vd, dev(token_seq.astype(np.int32)),
                            dev(token_pos.astype(np.int32)), bt, self.kc, self.kp, self.vc,
                            self.vp, err=self.err, tok_stride=tok_stride)
        oerr = 0
        if oracle_too:
            oerr = oracle.quantize_append(self.orc, k.view(np.uint16), v.view(np.uint16),
                                          token_seq, token_pos, block_table, self.okc,
                                          self.okp_pool(), self.ovc, self.ovp,
                                          tok_stride=tok_stride)
        torch.cuda.synchronize()
        return int(self.err.item()), oerr

    def assert_pools_equal(self):
        """Bit-exact comparison of codes and params (all bytes, untouched ones too)."""
        for g, o in ((self.kc, self.okc), (self.vc, self.ovc)):
            gh = g.cpu().numpy()
            if not np.array_equal(gh, o):
                bad = np.argwhere(gh != o)
                raise AssertionError(f"code bytes differ at {len(bad)} places, first {bad[:5]}")
        for g, o in ((self.kp, self.okp), (self.vp, self.ovp)):
            gh = g.cpu().numpy().view(o.dtype).reshape(o.shape)
            if not np.array_equal(gh, o):
                bad = np.argwhere(gh != o)
                raise AssertionError(f"param words differ at {len(bad)} places, first {bad[:5]}")

    def oracle_attention(self, q, seq_lens, max_seq_len, block_table, sm_scale):
        # the C ABI takes sm_scale as binary32: the oracle gets that same value
        return oracle.paged_decode_attn(self.orc, q.view(np.uint16), seq_lens, max_seq_len,
                                        block_table, float(np.float32(sm_scale)), self.okc,
                                        self.okp, self.ovc, self.ovp)

    def gpu_attention(self, q, seq_lens, max_seq_len, block_table, sm_scale):
        self.err.zero_()
        out = kvq.paged_decode_attn(self.gpu, dev(q), dev(seq_lens.astype(np.int32)), max_seq_len,
                                    dev(block_table.astype(np.int32)), self.kc, self.kp, self.vc,
                                    self.vp, sm_scale=sm_scale, err=self.err)
        torch.cuda.synchronize()
        return out.cpu().numpy().astype(np.float64), int(self.err.item())


def fill_workload(w, seqs=None, layer=0, oracle_too=True, fill=0xAA, fmt=kvq.FMT_INT4,
                  levels=None):
    """Pair cache holding the workload's cached tokens of the given sequences."""
    p = Pair.for_workload(w, fill, fmt, levels)
    k, v, ts, tp = w.prefill_tokens(seqs, layer)
    e, oe = p.append(k, v, ts, tp, w.block_table, oracle_too=oracle_too)
    assert e == 0 and oe == 0
    return p, (k, v, ts, tp)


def fused_step_vs_oracle(p, k_new, v_new, lens, table, q, sm_scale):
    """kvq_decode_step on p's GPU pools; the oracle's append of the same new
    tokens (token_seq = s, token_pos = lens[s] - 1; sequences with lens 0 skip)
    followed by its attention on p's oracle pools. Returns (GPU out, oracle
    out, GPU flags, oracle flags); the caller compares pools and outputs."""
    L = int(lens.max())
    S = len(lens)
    keep = lens >= 1
    ts = np.where(keep, np.arange(S, dtype=np.int32), -1).astype(np.int32)
    tp = np.maximum(lens - 1, 0).astype(np.int32)
    p.err.zero_()
    out = kvq.decode_step(p.gpu, dev(q), dev(k_new), dev(v_new), dev(lens.astype(np.int32)), L,
                          dev(table.astype(np.int32)), p.kc, p.kp, p.vc, p.vp, sm_scale=sm_scale,
                          err=p.err)
    torch.cuda.synchronize()
    oe = oracle.quantize_append(p.orc, k_new.view(np.uint16), v_new.view(np.uint16), ts, tp, table,
                                p.okc, p.okp_pool(), p.ovc, p.ovp)
    ref, oe2 = p.oracle_attention(q, lens, L, table, sm_scale)
    return out.cpu().numpy().astype(np.float64), ref, int(p.err.item()), oe | oe2
