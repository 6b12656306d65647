"""GPU parity of the further rotation kinds against the oracle:
IsoQuant-Fast (page "IsoQuant: Hardware-Aligned SO(4) Isoclinic Rotations for
LLM KV Cache Compression", Abstract: one isoclinic factor, v -> qL v), the
full map folded into one 4x4 matrix per block (same page: the map is linear),
and the randomised-sign Hadamard (channels flipped by a fixed sign table, then
the block Hadamard). Codes, scales and page placement bit-exact in the bulk and the
small-batch append kernels and in the fused decode step; decode attention
within 2e-3; the un-rotated dense export against the oracle's."""

import math

import numpy as np
import pytest
import torch

import oracle
from bit_rotated_kv_block_b200 import kvq, workloads
from gpu_helpers import Pair, dev, fill_workload, fused_step_vs_oracle

pytestmark = pytest.mark.gpu

TOL = 2e-3

KINDS = [(workloads.ROT_QUAT_FAST, 0, 128), (workloads.ROT_HADAMARD_SIGNED, 64, 128),
         (workloads.ROT_HADAMARD_SIGNED, 128, 128), (workloads.ROT_QUAT_FAST, 0, 256),
         (workloads.ROT_HADAMARD_SIGNED, 256, 256), (workloads.ROT_QUAT_MAT, 0, 128),
         (workloads.ROT_QUAT_MAT, 0, 256)]


def workload(kind, b, d):
    if d == 128:
        w = workloads.llama8b(S=5, ctx=900, spare_pages=8)
    else:
        w = workloads.ragged256(S=5, lo=300, hi=1500)
    w.rot_kind, w.rot_block = kind, b
    w.quat = (workloads.random_quaternions(11, d)
              if kind in (workloads.ROT_QUAT_FAST, workloads.ROT_QUAT_MAT)
              else workloads.random_signs(12, d))
    return w


@pytest.mark.parametrize("kind,b,d", KINDS)
def test_append_decode_step_and_export(kind, b, d):
    w = workload(kind, b, d)
    p, _ = fill_workload(w)  # bulk kernel (more than 8192 rows)
    p.assert_pools_equal()
    sm = 1 / math.sqrt(d)
    L = int(w.seq_lens.max())
    out, e = p.gpu_attention(w.queries(), w.seq_lens, L, w.block_table, sm)
    ref, oe = p.oracle_attention(w.queries(), w.seq_lens, L, w.block_table, sm)
    assert e == 0 and oe == 0
    assert np.max(np.abs(out - ref)) <= TOL
    # dense export, un-rotated, against the oracle's (binary32 arithmetic on
    # the device, double in the oracle)
    lens = dev(w.seq_lens)
    xg = kvq.dequantize_pages(p.gpu, lens, L, dev(w.block_table), p.kc, p.kp, unrotate=True)
    xo, _ = oracle.dequantize_pages(p.orc, w.seq_lens, L, w.block_table, p.okc,
                                    p.okp.reshape(p.orc.NP, p.orc.H, p.orc.P, 2), unrotate=True)
    xg = xg.cpu().numpy()
    mask = np.arange(L)[None, :] < w.seq_lens[:, None]
    assert np.max(np.abs(xg[mask] - xo[mask])) <= 1e-4 * max(1.0, np.abs(xo[mask]).max())
    # fused step (small-batch rows of the new tokens, then attention)
    k_new, v_new, _, _ = w.step_tokens(0)
    lens1 = (w.seq_lens + 1).astype(np.int32)
    out1, ref1, e, oe = fused_step_vs_oracle(p, k_new, v_new, lens1, w.block_table,
                                             w.queries(1), sm)
    assert e == 0 and oe == 0
    p.assert_pools_equal()
    assert np.max(np.abs(out1 - ref1)) <= TOL
