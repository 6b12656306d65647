"""GPU parity of kvq_dequantize_pages: the rotated-basis export is bit-exact
(c * s16 + m16 rounded once to binary32), the un-rotated export matches the
oracle's double-precision inverse rotation to binary32 rounding, and the
prefill workload's reconstruction MSE per Hadamard block size agrees with the
oracle's to 1e-6 relative."""

import numpy as np
import pytest
import torch

import oracle
from bit_rotated_kv_block_b200 import kvq, workloads
from gpu_helpers import dev, fill_workload

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,rot", [("tiny", workloads.ROT_HADAMARD),
                                      ("ragged", workloads.ROT_QUAT),
                                      ("ragged", workloads.ROT_HADAMARD)])
def test_export_matches_oracle(name, rot):
    if name == "tiny":
        w = workloads.tiny()
        seqs = None
    else:
        w = workloads.ragged256(rot_kind=rot, S=6, lo=20, hi=300)
        seqs = None
    p, _ = fill_workload(w, seqs=seqs)
    L = w.max_seq_len + 3
    lens = w.seq_lens
    for unrot in (0, 1):
        for f32 in (1, 0):
            sentinel = -7.0
            out = torch.full((w.S, L, w.H, w.d), sentinel, device="cuda",
                             dtype=torch.float32 if f32 else torch.float16)
            kvq.dequantize_pages(p.gpu, dev(lens), L, dev(w.block_table), p.kc, p.kp,
                                 unrotate=unrot, out_fp32=f32, out=out, err=p.err)
            torch.cuda.synchronize()
            got = out.cpu().numpy()
            ref, oe = oracle.dequantize_pages(p.orc, lens, L, w.block_table, p.okc, p.okp,
                                              unrot, f32)
            assert oe == 0 and int(p.err.item()) == 0
            for s in range(w.S):
                n = int(lens[s])
                g_s = got[s, :n].astype(np.float64) if f32 else got[s, :n].astype(np.float64)
                r_s = ref[s, :n] if f32 else ref[s, :n].view(np.float16).astype(np.float64)
                if unrot:
                    tol = 1e-6 * max(1.0, np.max(np.abs(r_s))) if f32 else None
                    if f32:
                        assert np.max(np.abs(g_s - r_s)) <= tol
                    else:
                        # binary16 rounding of the value plus the binary32
                        # inverse rotation's error, which scales with the
                        # row's magnitude rather than the element's
                        row = np.max(np.abs(r_s), axis=-1, keepdims=True)
                        assert np.all(np.abs(g_s - r_s) <= 2 ** -10 * np.abs(r_s) + 2e-6 * row + 2 ** -24)
                else:
                    assert np.array_equal(g_s, r_s)
                assert np.all(got[s, n:] == sentinel)


@pytest.mark.parametrize("b", [16, 32, 64, 128, 0])
def test_prefill_reconstruction_mse(b):
    # one full layer (65536 tokens x 8 heads) per block size
    w = workloads.prefill(rot_block=b)
    p, (k, v, ts, tp) = fill_workload(w)
    L = w.max_seq_len
    out = kvq.dequantize_pages(p.gpu, dev(w.seq_lens), L, dev(w.block_table), p.kc, p.kp,
                               unrotate=True)
    torch.cuda.synchronize()
    g = out.cpu().numpy().astype(np.float64)
    x = k.astype(np.float64).reshape(w.S, L, w.H, w.d)
    mse_gpu = float(np.mean((g - x) ** 2))
    ref, _ = oracle.dequantize_pages(p.orc, w.seq_lens, L, w.block_table, p.okc, p.okp, 1, 1)
    mse_orc = float(np.mean((ref.astype(np.float64) - x) ** 2))
    assert abs(mse_gpu - mse_orc) <= 1e-6 * mse_orc
