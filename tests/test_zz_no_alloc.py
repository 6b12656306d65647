"""The allocation-free decode entry point (kvq_paged_decode_attn_noalloc),
called through the C ABI, against the regular entry point.

Some callers cannot allocate device memory on their serving path (a
pre-planned engine whose allocator is closed after start-up, a plug-in inside
a framework that owns all device memory, code that must avoid the device
synchronisation of cudaMalloc). For them the library keeps its decode scratch
in a fixed 16 MiB device array. Both entry points run the same kernel with the
same plan on the same inputs, so their outputs must be equal bit for bit; one
case is also checked against the oracle. This file is collected last so that a
run stopping at the first failure has already run every other test; it builds
its own inputs so it also passes alone in a fresh process.
"""

import math

import numpy as np
import pytest
import torch

from bit_rotated_kv_block_b200 import kvq, workloads
from gpu_helpers import fill_workload

pytestmark = pytest.mark.gpu

TOL = 2e-3  # the attention tolerance of the other decode tests (oracle check)


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _workload(name, S):
    if name == "llama8b":
        return workloads.llama8b(S=S, ctx=1500)
    return workloads.ragged256(S=S, lo=100, hi=3000)


def _both_entries(w, p, calls=2):
    """The workspace entry once, the no-alloc entry ``calls`` times in a row."""
    q = _dev(w.queries())
    lens, bt = _dev(w.seq_lens), _dev(w.block_table)
    L = int(w.seq_lens.max())
    sm = 1 / math.sqrt(w.d)
    ref = kvq.paged_decode_attn(p.gpu, q, lens, L, bt, p.kc, p.kp, p.vc, p.vp, sm_scale=sm)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = []
    for _ in range(calls):  # later calls run on the scratch the earlier ones left behind
        outs.append(kvq.paged_decode_attn_noalloc(p.gpu, q, lens, L, bt, p.kc, p.kp, p.vc, p.vp,
                                                  sm_scale=sm, err=err))
        torch.cuda.synchronize()
    assert int(err.item()) == 0
    return ref, outs


@pytest.mark.parametrize("name", ["llama8b", "ragged256"])
def test_noalloc_equals_workspace_entry_two_calls(name):
    w = _workload(name, 8 if name == "llama8b" else 6)
    p, _ = fill_workload(w, oracle_too=(name == "llama8b"))
    ref, outs = _both_entries(w, p)
    for o in outs:
        assert torch.equal(o, ref)
    if name == "llama8b":
        # and the shared result against the oracle, within the attention bound
        orc, oe = p.oracle_attention(w.queries(), w.seq_lens, int(w.seq_lens.max()),
                                     w.block_table, 1 / math.sqrt(w.d))
        assert oe == 0
        assert np.max(np.abs(outs[-1].cpu().numpy().astype(np.float64) - orc)) <= TOL


def test_noalloc_after_calls_of_other_sizes():
    # the split counters sit at the start of the scratch and the partial
    # results right after them, at an offset that depends on the number of
    # (sequence, KV head) pairs; a call with fewer pairs leaves partial results
    # where a later call with more pairs keeps its counters. Each call must
    # clear its counters first: small -> large -> small, every result exact.
    small = workloads.llama8b(S=3, ctx=900)
    large = workloads.llama8b(S=40, ctx=300)
    ps, _ = fill_workload(small, oracle_too=False)
    pl, _ = fill_workload(large, oracle_too=False)
    for w, p in ((small, ps), (large, pl), (small, ps)):
        ref, outs = _both_entries(w, p, calls=1)
        assert torch.equal(outs[0], ref)


def test_noalloc_rejects_sizes_beyond_the_scratch():
    cache = kvq.Cache(128, 8, 16, 64, kvq.ROT_HADAMARD, 128)
    need = kvq.decode_workspace_bytes(cache, 4096, 64, 1 << 16)
    assert need > (16 << 20)
    q = torch.zeros((4096, 64, 128), dtype=torch.float16, device="cuda")
    lens = torch.zeros(4096, dtype=torch.int32, device="cuda")
    bt = torch.zeros((4096, 4096), dtype=torch.int32, device="cuda")
    kc, kp = cache.new_pools(fill=0)
    with pytest.raises(kvq.KvqError) as ei:
        kvq.paged_decode_attn_noalloc(cache, q, lens, 1 << 16, bt, kc, kp, kc, kp)
    assert ei.value.status == 4  # KVQ_ERR_WORKSPACE, nothing launched
