"""The allocation-free decode entry point (kvq_paged_decode_attn_noalloc),
called through the C ABI, against the regular entry point.

Some callers cannot allocate device memory on their serving path (a
pre-planned engine whose allocator is closed after start-up, a plug-in inside
a framework that owns all device memory, code that must avoid the device
synchronisation of cudaMalloc). For them the library keeps its decode scratch
in a fixed 16 MiB device array. This file is collected last so that a run
stopping at the first failure has already run every other test; it builds its
own inputs so it also passes alone in a fresh process.
"""

import math

import numpy as np
import pytest
import torch

from bit_rotated_kv_block_b200 import kvq, workloads

pytestmark = pytest.mark.gpu

TOL = 2e-3  # the attention tolerance the other decode tests use


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _filled(w, seqs):
    cache = kvq.Cache(w.d, w.H, w.P, w.NP, w.rot_kind, w.rot_block, w.quat)
    kc, kp = cache.new_pools(fill=0)
    vc, vp = cache.new_pools(fill=0)
    k, v, ts, tp = w.prefill_tokens(seqs)
    kvq.quantize_append(cache, _dev(k), _dev(v), _dev(ts), _dev(tp), _dev(w.block_table), kc, kp,
                        vc, vp)
    return cache, (kc, kp, vc, vp)


@pytest.mark.parametrize("name", ["llama8b", "ragged256"])
def test_noalloc_matches_workspace_entry_two_calls(name):
    if name == "llama8b":
        w = workloads.llama8b(S=8, ctx=1500)
        seqs = list(range(w.S))
    else:
        w = workloads.ragged256(S=6, lo=100, hi=3000)
        seqs = list(range(w.S))
    cache, (kc, kp, vc, vp) = _filled(w, seqs)
    q = _dev(w.queries())
    lens, bt = _dev(w.seq_lens), _dev(w.block_table)
    L = int(w.seq_lens.max())
    sm = 1 / math.sqrt(w.d)
    ref = kvq.paged_decode_attn(cache, q, lens, L, bt, kc, kp, vc, vp, sm_scale=sm)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = []
    for _ in range(2):  # the second call runs on the scratch the first left behind
        outs.append(kvq.paged_decode_attn_noalloc(cache, q, lens, L, bt, kc, kp, vc, vp,
                                                  sm_scale=sm, err=err))
        torch.cuda.synchronize()
    assert int(err.item()) == 0
    for o in outs:
        assert torch.isfinite(o).all()
        assert float((o - ref).abs().max()) <= TOL


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
