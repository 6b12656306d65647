"""GPU parity of the 2-bit, 3-bit and level-table cache formats (kvq.h,
KVQ_FMT_INT2 / INT3 / LUT4) against the oracle.

IsoQuant (page "IsoQuant: Hardware-Aligned SO(4) Isoclinic Rotations for LLM
KV Cache Compression", Abstract: bit widths {2, 3, 4}) and UltraQuant (page
"UltraQuant: 4-bit KV caching for long agents", method section: a calibrated
16-entry table in place of the uniform levels). Codes, parameters and page
placement bit-exact from the tiled and row append kernels and the fused
step; the dense export exact in the rotated basis; decode attention (QK on
tcgen05 integer MMA, PV on f16 tensor cores) within 2e-3 of the oracle.
"""

import math

import numpy as np
import pytest

import oracle
from bit_rotated_kv_block_b200 import calibrate, kvq, workloads
from gpu_helpers import Pair, dev, fill_workload, fused_step_vs_oracle

pytestmark = pytest.mark.gpu

TOL = 2e-3


def table_levels():
    """A level table calibrated on synthetic rotated rows (Hadamard b 64)."""
    g = np.random.default_rng(0)
    return calibrate.calibrate_levels(g.standard_normal((2000, 128)), 64)


def workload(rot, b, S=5, ctx=900):
    w = workloads.llama8b(S=S, ctx=ctx, spare_pages=8)
    w.rot_kind, w.rot_block = rot, b
    w.quat = workloads.random_quaternions(3, w.d) if rot == workloads.ROT_QUAT else None
    return w


CASES = [(kvq.FMT_INT2, workloads.ROT_HADAMARD, 64), (kvq.FMT_INT3, workloads.ROT_HADAMARD, 64),
         (kvq.FMT_LUT4, workloads.ROT_HADAMARD, 64), (kvq.FMT_INT3, workloads.ROT_QUAT, 0),
         (kvq.FMT_INT2, workloads.ROT_HADAMARD, 128), (kvq.FMT_LUT4, workloads.ROT_NONE, 0)]


@pytest.mark.parametrize("fmt,rot,b", CASES)
def test_append_export_decode_and_step(fmt, rot, b):
    lv = table_levels() if fmt == kvq.FMT_LUT4 else None
    w = workload(rot, b)
    p, _ = fill_workload(w, fmt=fmt, levels=lv)  # tiled kernel
    p.assert_pools_equal()
    L = int(w.seq_lens.max())
    sm = 1 / math.sqrt(w.d)
    lens, bt = dev(w.seq_lens), dev(w.block_table)
    xg = kvq.dequantize_pages(p.gpu, lens, L, bt, p.kc, p.kp, unrotate=False).cpu().numpy()
    xo, _ = oracle.dequantize_pages(p.orc, w.seq_lens, L, w.block_table, p.okc, p.okp, False)
    mask = np.arange(L)[None, :] < w.seq_lens[:, None]
    assert np.array_equal(xg[mask], xo[mask])
    out, e = p.gpu_attention(w.queries(), w.seq_lens, L, w.block_table, sm)
    ref, oe = p.oracle_attention(w.queries(), w.seq_lens, L, w.block_table, sm)
    assert e == 0 and oe == 0
    assert np.max(np.abs(out - ref)) <= TOL
    k_new, v_new, _, _ = w.step_tokens(0)
    lens1 = (w.seq_lens + 1).astype(np.int32)
    out1, ref1, e, oe = fused_step_vs_oracle(p, k_new, v_new, lens1, w.block_table,
                                             w.queries(1), sm)
    assert e == 0 and oe == 0
    p.assert_pools_equal()
    assert np.max(np.abs(out1 - ref1)) <= TOL


@pytest.mark.parametrize("fmt", [kvq.FMT_INT2, kvq.FMT_INT3, kvq.FMT_LUT4])
def test_rows_kernel_and_gqa8_ragged(fmt):
    lv = table_levels() if fmt == kvq.FMT_LUT4 else None
    # small batch: the row kernel (ragged positions, a skipped token, a bad page)
    w = workload(workloads.ROT_HADAMARD, 64, S=4, ctx=300)
    p = Pair.for_workload(w, fmt=fmt, levels=lv)
    k, v, ts, tp = w.prefill_tokens()
    sel = np.arange(0, len(ts), 7)[:400]
    ts2, tp2 = ts[sel].copy(), tp[sel].copy()
    ts2[5] = -1
    table = w.block_table.copy()
    table[2, 3] = w.NP + 5
    e, oe = p.append(k[sel], v[sel], ts2, tp2, table)
    assert e == oe and (e & kvq.ERRF_PAGE)
    p.assert_pools_equal()
    # long-context shaped (G 8, page 32): lengths 0, 1, a tile tail, several tiles
    w = workloads.long70b(S=4, ctx=700)
    w.seq_lens = np.array([0, 1, 129, 700], np.int32)
    p, _ = fill_workload(w, fmt=fmt, levels=lv)
    p.assert_pools_equal()
    sm = 1 / math.sqrt(w.d)
    L = int(w.seq_lens.max())
    out, e = p.gpu_attention(w.queries(), w.seq_lens, L, w.block_table, sm)
    ref, oe = p.oracle_attention(w.queries(), w.seq_lens, L, w.block_table, sm)
    assert e == 0 and oe == 0
    assert np.all(out[0] == 0)
    assert np.max(np.abs(out - ref)) <= TOL


def test_llama8b_full_size_lut4_step():
    # the bench's workload and launch configuration in the table format
    lv = table_levels()
    w = workloads.llama8b()
    p, _ = fill_workload(w, fmt=kvq.FMT_LUT4, levels=lv)
    k_new, v_new, _, _ = w.step_tokens(0)
    lens = (w.seq_lens + 1).astype(np.int32)
    out, ref, e, oe = fused_step_vs_oracle(p, k_new, v_new, lens, w.block_table, w.queries(),
                                           1 / math.sqrt(w.d))
    assert e == 0 and oe == 0
    p.assert_pools_equal()
    assert np.max(np.abs(out - ref)) <= TOL


def test_format_arguments_are_checked():
    # host-side rejections (status 1 invalid argument, 2 unsupported), nothing
    # launched: an unknown format, the formats other than INT4 at head_dim 256,
    # the table format without its table and a table given to another format
    w = workload(workloads.ROT_HADAMARD, 64, S=1, ctx=32)
    k, v, ts, tp = w.prefill_tokens()
    for fmt, d, lv, want in ((7, 128, None, 1),
                             (kvq.FMT_INT3, 256, None, 2),
                             (kvq.FMT_LUT4, 128, None, 1),
                             (kvq.FMT_INT2, 128, np.arange(16, dtype=np.float32),
                              1)):
        c = kvq.Cache(d, w.H, w.P, w.NP, workloads.ROT_HADAMARD, 64, fmt=fmt if fmt != 7 else 0,
                      levels=lv)
        c.desc.format = fmt
        kc, kp = c.new_pools(fill=0)
        kk = dev(np.zeros((len(ts), w.H, d), np.float16))
        with pytest.raises(kvq.KvqError) as ei:
            kvq.quantize_append(c, kk, kk, dev(ts), dev(tp), dev(w.block_table), kc, kp, kc, kp)
        assert ei.value.status == want
