"""The ragged head_dim-256 workload at its stated size, through the C ABI,
against the oracle: 128 sequences with lengths uniform in [512, 16384]
(about 1.08 M cached tokens), 4 KV heads, 16 query heads, per-channel scales
log-uniform in [0.1, 20], page 16, with the block-diagonal Hadamard rotation
(block 256) and with the per-4-channel quaternion rotation (page "IsoQuant:
Hardware-Aligned SO(4) Isoclinic Rotations for LLM KV Cache Compression",
Abstract). Every launch has the real plan of that size (128 sequences in one
decode launch):

* the bulk fill of every sequence: codes, scales and minima bit-exact;
* decode attention of all 128 x 16 query heads within 2e-3 of the oracle;
* one fused decode step (new token of every sequence, then attention): pools
  bit-exact and every output within 2e-3 of the oracle.
"""

import math

import numpy as np
import pytest

from bit_rotated_kv_block_b200 import workloads
from gpu_helpers import fill_workload, fused_step_vs_oracle

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module", params=[workloads.ROT_HADAMARD, workloads.ROT_QUAT],
                ids=["hadamard256", "quaternion"])
def full(request):
    w = workloads.ragged256(rot_kind=request.param)
    p, _ = fill_workload(w)
    yield w, p
    del p


def test_fill_all_sequences_bit_exact(full):
    w, p = full
    assert w.S == 128 and int(w.seq_lens.sum()) > 1_000_000
    p.assert_pools_equal()


def test_decode_all_sequences(full):
    w, p = full
    L = int(w.seq_lens.max())
    sm = 1 / math.sqrt(w.d)
    q = w.queries()
    out, e = p.gpu_attention(q, w.seq_lens, L, w.block_table, sm)
    ref, oe = p.oracle_attention(q, w.seq_lens, L, w.block_table, sm)
    assert e == 0 and oe == 0
    assert out.shape == (128, 16, 256)
    err = float(np.max(np.abs(out - ref)))
    assert err <= TOL, f"max abs error {err}"


def test_fused_step_all_sequences(full):
    # runs last for each rotation: it appends one token to every sequence
    w, p = full
    k_new, v_new, _, _ = w.step_tokens(0)
    lens = (w.seq_lens + 1).astype(np.int32)
    out, ref, e, oe = fused_step_vs_oracle(p, k_new, v_new, lens, w.block_table, w.queries(1),
                                           1 / math.sqrt(w.d))
    assert e == 0 and oe == 0
    p.assert_pools_equal()
    err = float(np.max(np.abs(out - ref)))
    assert err <= TOL, f"max abs error {err}"
