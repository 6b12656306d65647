"""GPU parity of the microscaled FP4 cache format (kvq.h, KVQ_FMT_MXFP4)
against the oracle.

UltraQuant (page "UltraQuant: 4-bit KV caching for long agents", method
section): FP4 KV tensors with UE8M0 group scales, FP8 queries, the matrix
cores' scaled multiply-accumulate. Codes and scale bytes bit-exact from the
tiled and the small-batch append kernels and from the fused decode step; the
dense export exact in binary32 (rotated basis) and within the un-rotation's
rounding otherwise; decode attention (QK on tcgen05 block-scaled MMA) within
2e-3 of the oracle, whose query is quantized to MX E4M3 the same way.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from bit_rotated_kv_block_b200 import kvq, workloads
from gpu_helpers import Pair, dev, fill_workload, fused_step_vs_oracle

pytestmark = pytest.mark.gpu

TOL = 2e-3
MX = kvq.FMT_MXFP4

ROTS = [(workloads.ROT_HADAMARD, 64), (workloads.ROT_HADAMARD, 128), (workloads.ROT_NONE, 0),
        (workloads.ROT_QUAT, 0), (workloads.ROT_HADAMARD_SIGNED, 64)]


def llama_small(rot, b, S=5, ctx=900):
    w = workloads.llama8b(S=S, ctx=ctx, spare_pages=8)
    w.rot_kind, w.rot_block = rot, b
    if rot in (workloads.ROT_QUAT, workloads.ROT_QUAT_FAST, workloads.ROT_QUAT_MAT):
        w.quat = workloads.random_quaternions(3, w.d)
    elif rot == workloads.ROT_HADAMARD_SIGNED:
        w.quat = workloads.random_signs(4, w.d)
    else:
        w.quat = None
    return w


@pytest.mark.parametrize("rot,b", ROTS)
def test_append_export_decode_and_step(rot, b):
    w = llama_small(rot, b)
    p, _ = fill_workload(w, fmt=MX)  # tiled kernel (more than 8192 rows)
    p.assert_pools_equal()
    L = int(w.seq_lens.max())
    sm = 1 / math.sqrt(w.d)
    # dense export: exact in the rotated basis
    lens, bt = dev(w.seq_lens), dev(w.block_table)
    xg = kvq.dequantize_pages(p.gpu, lens, L, bt, p.kc, p.kp, unrotate=False).cpu().numpy()
    xo, _ = oracle.dequantize_pages(p.orc, w.seq_lens, L, w.block_table, p.okc, p.okp, False)
    mask = np.arange(L)[None, :] < w.seq_lens[:, None]
    assert np.array_equal(xg[mask], xo[mask])
    xg = kvq.dequantize_pages(p.gpu, lens, L, bt, p.vc, p.vp, unrotate=True).cpu().numpy()
    xo, _ = oracle.dequantize_pages(p.orc, w.seq_lens, L, w.block_table, p.ovc, p.ovp, True)
    assert np.max(np.abs(xg[mask] - xo[mask])) <= 1e-4 * max(1.0, np.abs(xo[mask]).max())
    # decode attention
    out, e = p.gpu_attention(w.queries(), w.seq_lens, L, w.block_table, sm)
    ref, oe = p.oracle_attention(w.queries(), w.seq_lens, L, w.block_table, sm)
    assert e == 0 and oe == 0
    assert np.max(np.abs(out - ref)) <= TOL
    # fused step: the new token of every sequence through the step kernel
    k_new, v_new, _, _ = w.step_tokens(0)
    lens1 = (w.seq_lens + 1).astype(np.int32)
    out1, ref1, e, oe = fused_step_vs_oracle(p, k_new, v_new, lens1, w.block_table,
                                             w.queries(1), sm)
    assert e == 0 and oe == 0
    p.assert_pools_equal()
    assert np.max(np.abs(out1 - ref1)) <= TOL


def test_rows_kernel_bit_exact_and_flags():
    # a batch under 8192 rows goes to the row kernel: ragged positions, a
    # skipped token, a page outside the pool (flagged, nothing written)
    w = llama_small(workloads.ROT_HADAMARD, 64, S=4, ctx=300)
    p = Pair.for_workload(w, fmt=MX)
    k, v, ts, tp = w.prefill_tokens()
    sel = np.arange(0, len(ts), 7)[:400]
    ts2, tp2 = ts[sel].copy(), tp[sel].copy()
    ts2[5] = -1
    table = w.block_table.copy()
    table[2, 3] = w.NP + 5
    e, oe = p.append(k[sel], v[sel], ts2, tp2, table)
    assert e == oe and (e & kvq.ERRF_PAGE)
    p.assert_pools_equal()


def test_ragged_lengths_gqa8_page32():
    # long-context shaped (G 8, page 32): lengths 0, 1, a tile tail, several tiles
    w = workloads.long70b(S=4, ctx=700)
    w.seq_lens = np.array([0, 1, 129, 700], np.int32)
    p, _ = fill_workload(w, fmt=MX)
    p.assert_pools_equal()
    sm = 1 / math.sqrt(w.d)
    L = int(w.seq_lens.max())
    out, e = p.gpu_attention(w.queries(), w.seq_lens, L, w.block_table, sm)
    ref, oe = p.oracle_attention(w.queries(), w.seq_lens, L, w.block_table, sm)
    assert e == 0 and oe == 0
    assert np.all(out[0] == 0)
    assert np.max(np.abs(out - ref)) <= TOL


def test_invalid_page_in_decode_is_flagged_and_skipped():
    w = llama_small(workloads.ROT_HADAMARD, 64, S=3, ctx=400)
    p, _ = fill_workload(w, fmt=MX)
    table = w.block_table.copy()
    table[1, 2] = -7  # tokens 32..47 of sequence 1
    sm = 1 / math.sqrt(w.d)
    L = int(w.seq_lens.max())
    out, e = p.gpu_attention(w.queries(), w.seq_lens, L, table, sm)
    ref, oe = p.oracle_attention(w.queries(), w.seq_lens, L, table, sm)
    assert (e & kvq.ERRF_PAGE) and (oe & kvq.ERRF_PAGE)
    assert np.max(np.abs(out - ref)) <= TOL


def test_llama8b_full_size_decode():
    # the bench's workload and launch configuration: 32 sequences x 4097
    # cached tokens after one fused step; every (sequence, query head) against
    # the oracle
    w = workloads.llama8b()
    p, _ = fill_workload(w, fmt=MX)
    k_new, v_new, _, _ = w.step_tokens(0)
    lens = (w.seq_lens + 1).astype(np.int32)
    out, ref, e, oe = fused_step_vs_oracle(p, k_new, v_new, lens, w.block_table, w.queries(),
                                           1 / math.sqrt(w.d))
    assert e == 0 and oe == 0
    p.assert_pools_equal()
    assert np.max(np.abs(out - ref)) <= TOL
