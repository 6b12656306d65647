"""GPU parity of the full-precision baseline kvq_paged_decode_attn_fp16
against the oracle's double-precision attention over the same binary16 pages
(no quantization, no rotation): max |out - oracle| <= 2e-3."""

import math

import numpy as np
import pytest
import torch

import oracle
from bit_rotated_kv_block_b200 import kvq, workloads

pytestmark = pytest.mark.gpu

TOL = 2e-3


def fp16_pages(w, k, v, ts, tp):
    """Scatter token rows into [NP][H][P][d] binary16 pools (test plumbing)."""
    kp = np.zeros((w.NP, w.H, w.P, w.d), np.float16)
    vp = np.zeros((w.NP, w.H, w.P, w.d), np.float16)
    page = w.block_table[ts, tp // w.P]
    slot = tp % w.P
    kp[page, :, slot, :] = k
    vp[page, :, slot, :] = v
    return kp, vp


def run(w, lens, L, table=None, kp=None, vp=None, q=None):
    table = w.block_table if table is None else table
    if kp is None:
        k, v, ts, tp = w.prefill_tokens()
        kp, vp = fp16_pages(w, k, v, ts, tp)
    q = w.queries() if q is None else q
    sm = 1 / math.sqrt(w.d)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    c = kvq.Cache(w.d, w.H, w.P, w.NP, workloads.ROT_NONE, 0)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = kvq.paged_decode_attn_fp16(c, dev(q), dev(np.asarray(lens, np.int32)), L, dev(table),
                                     dev(kp), dev(vp), sm_scale=sm, err=err)
    torch.cuda.synchronize()
    ref, oe = oracle.paged_decode_attn_fp16(w.d, w.H, w.P, w.NP, q.view(np.uint16), lens, L,
                                           table, float(np.float32(sm)), kp.view(np.uint16),
                                           vp.view(np.uint16))
    assert int(err.item()) == oe
    e = float(np.max(np.abs(out.cpu().numpy().astype(np.float64) - ref))) if ref.size else 0.0
    assert e <= TOL, f"max abs error {e}"
    return e


def test_tiny():
    w = workloads.tiny()
    run(w, w.seq_lens, 256)


def test_llama_shaped_small():
    # GQA 4, page 16, a x10 sink token and outlier channels, ragged last page
    w = workloads.llama8b(S=3, ctx=1000, spare_pages=4)
    run(w, w.seq_lens, int(w.seq_lens.max()))


def test_long70b_shaped_small():
    # GQA 8, page 32
    w = workloads.long70b(S=2, ctx=3000)
    run(w, w.seq_lens, int(w.seq_lens.max()))


def test_head_dim_256_ragged():
    w = workloads.ragged256(S=4, lo=100, hi=700, rot_kind=workloads.ROT_HADAMARD)
    run(w, w.seq_lens, int(w.seq_lens.max()))


def test_edges_empty_sequence_and_bad_page():
    w = workloads.llama8b(S=3, ctx=300, spare_pages=4)
    k, v, ts, tp = w.prefill_tokens()
    kp, vp = fp16_pages(w, k, v, ts, tp)
    lens = np.array([0, 300, 17], np.int32)
    table = w.block_table.copy()
    table[1, 3] = w.NP + 5  # page outside the pool: skipped and flagged
    run(w, lens, 300, table=table, kp=kp, vp=vp)
