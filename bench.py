"""Benchmark of the rotated INT4 paged KV-cache hot path on B200.

One step = one pass of the whole path over one batch of the Llama-3-8B-shaped
decode layer (32 sequences x 4096 cached tokens, 8 KV heads, 32 query heads,
head_dim 128, Hadamard block 64, page 16, shuffled block table): append one
new token per sequence (fused rotate -> INT4 -> pack -> page scatter), then
paged decode attention over the 4097 cached INT4 tokens -- both in one
kvq_decode_step launch. Inputs are seeded
synthetic draws of that shape (no dataset exists for this workload).

The device-timed region covers exactly --steps steps between a barrier and a
synchronize on both sides; consecutive steps alternate between two cache
replicas (2 x 143 MB > the 126 MB L2), so every step reads its pages from HBM.
Also measured (outside that region): the bulk prefill append of the same
layer (131072 tokens) in GB/s.

Multi-GPU: one process per GPU (torchrun); every rank runs an independent
shard of sequences (weak scaling, no collective on the data path); the
reported time is the max over ranks.

--impl reference times the CPU oracle (the only reference this method has) on
rank 0 on a bounded sample of the same workload.

Prints one JSON line.
"""

import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

WORKLOAD = "llama8b"
METRIC = "INT4 paged decode-attn tokens/s (append + decode step, one layer)"
UNIT = "tokens/s"
BYTES_PER_TOKEN_HEAD = 136  # decode: 2 * (64 code bytes + 4 param bytes), head_dim 128
APPEND_BYTES_PER_TOKEN_HEAD = 648  # append: 2 * 256 B read + 2 * 68 B written
NOMINAL_HBM_GBS = 8000.0  # the B200's nominal HBM bandwidth, for the second set of fractions


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the per-workload records (long-context decode, prefill sweep, "
                         "ragged head_dim-256 step) that a one-GPU run adds to the line")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work")
    ap.add_argument("--compare", action="store_true",
                    help="print one JSON line with the baseline comparisons (long-context INT4 with "
                         "and without rotation vs the binary16 cache; prefill append per Hadamard "
                         "block with reconstruction MSE) and exit")
    ap.add_argument("--profile-case", choices=["append", "decode", "decode-mx", "decode-int3",
                                               "decode-lut4"], default=None,
                    help="run a short fixed case for an ncu capture (4 launches) and exit")
    ap.add_argument("--profile-block", type=int, default=128,
                    help="Hadamard block size of the append profile case (0: no rotation)")
    ap.add_argument("--profile-workload", choices=["llama8b", "long70b"], default="llama8b",
                    help="workload of the decode profile case")
    return ap.parse_args()


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def shard_seed(seed, rank):
    """Seed of rank ``rank``'s shard: every rank draws its own sequences."""
    return seed + 1000 * rank


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world, device):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, world, device):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"kvq_clocks_rank{index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        if not rows:
            return None
        sm = np.array([float(r[1]) for r in rows if r[1].replace(".", "").isdigit()])
        mx = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        loaded = sm[sm > 0.5 * mx] if sm.size else sm
        med = float(np.median(loaded)) if loaded.size else (float(np.median(sm)) if sm.size else None)
        return {"sm_mhz": med, "sm_max_mhz": mx, "reasons": reasons, "samples": int(sm.size)}


# ---------------------------------------------------------------- peaks

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def source_code_hash(path):
    """sha256 (16 hex digits) of a C/CUDA source with its comments, blank lines
    and indentation removed: it changes with the code, not with its comments."""
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    code = "\n".join(" ".join(ln.split()) for ln in text.splitlines() if ln.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def kernel_traffic(kernel):
    """DRAM bytes per launch from the committed ncu summary, valid only while
    the kernel's code is unchanged since the capture (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path)).get(kernel)
    if not d:
        return None
    h = source_code_hash(os.path.join(ROOT, d["source"]))
    return float(d["bytes_per_launch"]) if h == d["source_code_sha256_16"] else None


# ---------------------------------------------------------------- our arm

def run_ours(args, world, rank, local):
    from bit_rotated_kv_block_b200 import kvq, workloads
    from bit_rotated_kv_block_b200 import build as kbuild

    if not torch.cuda.is_available():
        # the measured path is the CUDA library; there is no CPU fallback
        raise SystemExit("bench.py: the INT4 KV-cache path needs a CUDA GPU; "
                         "--impl reference times the CPU oracle")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if rank == 0 or not os.path.exists(kbuild.LIB):
        kbuild.build()
    barrier(world)
    kvq.lib()
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(device)

    # each rank owns an independent shard of 32 sequences (seeded per rank)
    w = workloads.llama8b(seed=shard_seed(args.seed, rank))
    S, H, Hq, d, ctx = w.S, w.H, w.Hq, w.d, int(w.seq_lens[0])
    k, v, ts, tp = w.prefill_tokens()
    K, V, TS, TP = dev(k), dev(v), dev(ts), dev(tp)
    BT = dev(w.block_table)
    caches = []
    for rep in range(2):
        c = kvq.Cache(w.d, w.H, w.P, w.NP, w.rot_kind, w.rot_block)
        kc, kp = c.new_pools(device=device, fill=0)
        vc, vp = c.new_pools(device=device, fill=0)
        kvq.quantize_append(c, K, V, TS, TP, BT, kc, kp, vc, vp)
        caches.append((c, kc, kp, vc, vp))
    torch.cuda.synchronize()

    # bulk prefill append throughput (131072 tokens, inputs 268 MB > L2)
    c0, kc0, kp0, vc0, vp0 = caches[0]
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(8)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(8)]
    for i in range(3):
        kvq.quantize_append(c0, K, V, TS, TP, BT, kc0, kp0, vc0, vp0)
    for i in range(8):
        e0[i].record()
        kvq.quantize_append(c0, K, V, TS, TP, BT, kc0, kp0, vc0, vp0)
        e1[i].record()
    torch.cuda.synchronize()
    t_app = float(np.median([a.elapsed_time(b) for a, b in zip(e0, e1)])) * 1e-3
    app_bytes = len(ts) * H * APPEND_BYTES_PER_TOKEN_HEAD
    del K, V

    # step inputs: one new token per sequence at position ctx, and queries
    ks, vs, sts, stp = w.step_tokens(0)
    q = w.queries(0)
    lens = (w.seq_lens + 1).astype(np.int32)
    SK, SV, STS, STP, Q, LENS = dev(ks), dev(vs), dev(sts), dev(stp), dev(q), dev(lens)
    L = int(lens.max())
    out = torch.empty((S, Hq, d), dtype=torch.float32, device=device)
    ws = torch.zeros(kvq.decode_workspace_bytes(c0, S, Hq, L), dtype=torch.uint8, device=device)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream()
    # kvq_decode_step: the split kernel (new-token append and attention over
    # page ranges) and the merge kernel of the splits
    launches_per_step = 2

    def step(i):
        c, kc, kp, vc, vp = caches[i % 2]
        kvq.decode_step(c, Q, SK, SV, LENS, L, BT, kc, kp, vc, vp, out=out, workspace=ws, err=err)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    steps = args.steps
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    t0.record(stream)
    # the timed region holds nothing but the step kernels (a split and a merge
    # kernel per step, launched with programmatic serialization so each starts
    # while the previous one drains); its duration per step bounds the split
    # kernel's launch duration from above, so the roofline figure derived
    # from it is conservative
    for i in range(steps):
        c, kc, kp, vc, vp = caches[i % 2]
        kvq.decode_step(c, Q, SK, SV, LENS, L, BT, kc, kp, vc, vp, out=out, workspace=ws, err=err)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    elapsed = t0.elapsed_time(t1) * 1e-3
    t_dec = elapsed / steps
    assert int(err.item()) == 0, f"device error flags {int(err.item())}"

    elapsed_max = max_over_ranks(elapsed, world, device)
    units = sum_over_ranks(float(S * steps), world, device)
    value = units / elapsed_max
    ms_per_step = elapsed_max / steps * 1e3

    # end to end through the public API with host buffers: pinned inputs in,
    # result out, every step
    # the step's inputs (new K and V rows, queries) travel in one pinned
    # buffer and one copy; the result comes back in one copy. As a serving
    # loop would, the copies run on their own streams (one per direction) and
    # overlap the neighbouring steps' kernels: inputs and outputs are double
    # buffered, step i reads input buffer i % 2 once its copy has landed and
    # its result leaves while step i + 1 runs
    nk, nv, nq = ks.size, vs.size, q.size
    hin = torch.empty(nk + nv + nq, dtype=torch.float16).pin_memory()
    hin[:nk] = torch.from_numpy(ks.reshape(-1))
    hin[nk:nk + nv] = torch.from_numpy(vs.reshape(-1))
    hin[nk + nv:] = torch.from_numpy(q.reshape(-1))
    dins = [torch.empty(nk + nv + nq, dtype=torch.float16, device=device) for _ in range(2)]
    views = [(dn[:nk].view(ks.shape), dn[nk:nk + nv].view(vs.shape), dn[nk + nv:].view(q.shape))
             for dn in dins]
    outs = [torch.empty((S, Hq, d), dtype=torch.float32, device=device) for _ in range(2)]
    houts = [torch.empty((S, Hq, d), dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d = hin.numel() * 2
    d2h = houts[0].numel() * 4
    e2e_steps = min(steps, 500)
    up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    issued = [False, False]

    def e2e_step(i):
        b = i % 2
        c, kc, kp, vc, vp = caches[b]
        with torch.cuda.stream(up):
            if issued[b]:
                up.wait_event(ev_done[b])  # step i - 2 has read this buffer
            dins[b].copy_(hin, non_blocking=True)
            ev_in[b].record(up)
        stream.wait_event(ev_in[b])
        if issued[b]:
            stream.wait_event(ev_out[b])  # step i - 2's result has left this buffer
        SKb, SVb, Qb = views[b]
        kvq.decode_step(c, Qb, SKb, SVb, LENS, L, BT, kc, kp, vc, vp, out=outs[b], workspace=ws,
                        err=err)
        ev_done[b].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(ev_done[b])
            houts[b].copy_(outs[b], non_blocking=True)
            ev_out[b].record(down)
        issued[b] = True

    for i in range(3):
        e2e_step(i)
    barrier(world)
    torch.cuda.synchronize()
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    ev_start = torch.cuda.Event()
    ev_start.record(stream)
    up.wait_event(ev_start)  # no copy of the timed steps starts before the region
    down.wait_event(ev_start)
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_event(ev_out[(e2e_steps - 1) % 2])  # the last result is on the host
    stream.wait_event(ev_out[e2e_steps % 2])
    a1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_t = max_over_ranks(a0.elapsed_time(a1) * 1e-3, world, device)
    e2e_value = sum_over_ranks(float(S * e2e_steps), world, device) / e2e_t

    if rank != 0:
        return None
    peak, peak_kind = measured_peaks()
    dec_bytes = S * L * H * BYTES_PER_TOKEN_HEAD
    achieved = dec_bytes / t_dec / 1e9
    traffic = kernel_traffic("decode_llama8b")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u4 codes / f16 params / f32 math",
        "data": "synthetic",
        "config": {"workload": "Llama-3-8B-shaped decode layer: 32 seqs x 4096 ctx (+1 appended),"
                               " 8 KV heads, 32 q heads, d 128, Hadamard b 64, page 16",
                   "global_batch": S * world, "seq_len": L, "parallelism": f"replicas x{world}",
                   "l2": "steps alternate between 2 cache replicas (2 x 143 MB > 126 MB L2)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "decode step (split kernel; per-step time incl. the merge kernel)",
                     "bytes_per_launch": dec_bytes, "peak_source": peak_kind,
                     "frac_nominal": achieved / NOMINAL_HBM_GBS},
        "append_prefill": {"gbs": app_bytes / t_app / 1e9, "frac": app_bytes / t_app / 1e9 / peak,
                           "frac_nominal": app_bytes / t_app / 1e9 / NOMINAL_HBM_GBS,
                           "us": t_app * 1e6, "bytes": app_bytes, "tokens": len(ts)},
        "decode": {"us": t_dec * 1e6, "kv_tokens_per_s": S * L / t_dec,
                   "gbs": achieved},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * steps,
        "clocks": clk,
    }
    if world == 1 and not args.no_workloads:
        # outside the timed region: the other workloads' kernels, each timed alone
        del caches, ws
        torch.cuda.empty_cache()
        line["workloads"] = workload_records(device, args.seed)
    return line, w


# ---------------------------------------------------------------- CPU oracle

def oracle_step_sample(w, n_heads_budget, seed_rank=0):
    """Set up the oracle's cache for one sequence; returns a closure that runs
    one bounded sample (the step append of that sequence's token and decode
    attention for ``n_heads_budget`` query heads) and the number of query
    tokens (in units of a full 32-head token) it covers."""
    import oracle
    s = 0
    k, v, ts, tp = w.prefill_tokens(seqs=[s])
    oc = oracle.Cache(w.d, w.H, w.P, w.NP, w.rot_kind, w.rot_block)
    kc, kp = oc.alloc_pools(0)
    vc, vp = oc.alloc_pools(0)
    oracle.quantize_append(oc, k.view(np.uint16), v.view(np.uint16), ts, tp, w.block_table,
                           kc, kp, vc, vp)
    ks, vs, sts, stp = w.step_tokens(0)
    q = w.queries(0)
    lens = np.array([int(w.seq_lens[s]) + 1], np.int32)
    nh = max(1, min(w.Hq, n_heads_budget))
    q_s = np.ascontiguousarray(q[s:s + 1, :nh])
    # attention over the first nh query heads: a cache view whose query-head
    # count is nh requires nh to be a multiple of H; round to whole groups
    G = w.Hq // w.H
    nkv = max(1, nh // G)
    nh = nkv * G
    q_s = np.ascontiguousarray(q[s:s + 1, :nh])
    oc_sub = oracle.Cache(w.d, nkv, w.P, w.NP, w.rot_kind, w.rot_block)
    kc_s = np.ascontiguousarray(kc[:, :nkv])
    kp_s = np.ascontiguousarray(kp[:, :nkv])
    vc_s = np.ascontiguousarray(vc[:, :nkv])
    vp_s = np.ascontiguousarray(vp[:, :nkv])

    def run():
        oracle.quantize_append(oc, ks[s:s + 1].view(np.uint16), vs[s:s + 1].view(np.uint16),
                               np.array([0], np.int32), stp[s:s + 1], w.block_table[s:s + 1],
                               kc, kp, vc, vp)
        oracle.paged_decode_attn(oc_sub, q_s.view(np.uint16), lens, int(lens[0]),
                                 w.block_table[s:s + 1], 1 / math.sqrt(w.d), kc_s, kp_s, vc_s,
                                 vp_s)

    return run, nh / w.Hq


def cpu_model():
    """The host CPU's model name (lscpu, else /proc/cpuinfo)."""
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            if line.startswith("Model name:"):
                return line.split(":", 1)[1].strip()
    except (OSError, subprocess.SubprocessError):
        pass
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def cpu_baseline(w, budget_s):
    """The oracle timed on the host cores on a bounded sample, with OpenMP on
    every core and again on one thread."""
    import oracle
    run, frac = oracle_step_sample(w, w.Hq)

    def timed(budget):
        t = time.perf_counter()
        run()
        one = time.perf_counter() - t
        reps = max(1, int(budget / max(one, 1e-3)))
        t = time.perf_counter()
        for _ in range(reps):
            run()
        return reps, time.perf_counter() - t

    cores = oracle.num_threads()
    reps, el = timed(budget_s)
    oracle.set_num_threads(1)
    try:
        reps1, el1 = timed(budget_s / 2)
    finally:
        oracle.set_num_threads(cores)
    return {"value": reps * frac / el, "unit": UNIT, "cores": cores,
            "value_1thread": reps1 * frac / el1, "cpu_model": cpu_model(),
            "kind": "oracle",
            "sample": f"{reps} (all cores) and {reps1} (1 thread) x (append of 1 token + decode "
                      f"attention of 1 sequence x {int(frac * w.Hq)} query heads over "
                      f"{int(w.seq_lens[0]) + 1} INT4 tokens), fp64 attention, OpenMP over heads"}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    import oracle
    from bit_rotated_kv_block_b200 import workloads
    w = workloads.llama8b(seed=args.seed)
    # size each step's sample so warmup + steps of oracle work take ~2 minutes
    budget = 120.0
    per_step = budget / max(1, args.steps + args.warmup)
    run_full, _ = oracle_step_sample(w, w.Hq)
    t = time.perf_counter()
    run_full()
    full = time.perf_counter() - t
    heads = int(max(w.Hq // w.H, min(w.Hq, w.Hq * per_step / max(full, 1e-6))))
    run, frac = oracle_step_sample(w, heads)
    for _ in range(args.warmup):
        run()
    t = time.perf_counter()
    for _ in range(args.steps):
        run()
    el = time.perf_counter() - t
    value = args.steps * frac / el
    sample = (f"per step: append of 1 token + decode attention of 1 sequence x "
              f"{int(round(frac * w.Hq))} query heads over {int(w.seq_lens[0]) + 1} tokens")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32 quantize / f64 attention (CPU oracle)", "data": "synthetic",
        "config": {"workload": "Llama-3-8B-shaped decode layer (bounded sample per step)",
                   "global_batch": 32, "seq_len": int(w.seq_lens[0]) + 1,
                   "parallelism": "rank 0 CPU"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def profile_case(which, block=128, workload="llama8b"):
    """Short cases for ncu captures, each well above L2 and well below a few GB:
    append = 4 bulk appends of one prefill layer (65536 tokens, Hadamard block
    `block`, 268 MB in, 71 MB out); decode = 4 decode calls of the
    Llama-3-8B-shaped layer (143 MB of INT4 pages) or of the long-context
    70B-shaped one (285 MB) after filling its cache with one append; decode-mx,
    decode-int3, decode-lut4 = the same decode calls over the microscaled FP4,
    3-bit and level-table caches."""
    from bit_rotated_kv_block_b200 import kvq, workloads
    torch.cuda.set_device(0)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    if which == "append":
        w = workloads.prefill(rot_block=block)
    else:
        w = workloads.long70b() if workload == "long70b" else workloads.llama8b()
    k, v, ts, tp = w.prefill_tokens()
    fmt = {"decode-mx": kvq.FMT_MXFP4, "decode-int3": kvq.FMT_INT3,
           "decode-lut4": kvq.FMT_LUT4}.get(which, kvq.FMT_INT4)
    levels = None
    if fmt == kvq.FMT_LUT4:
        from bit_rotated_kv_block_b200 import calibrate
        levels = calibrate.calibrate_levels(np.random.default_rng(77).standard_normal((4000, w.d)),
                                            w.rot_block)
    c = kvq.Cache(w.d, w.H, w.P, w.NP, w.rot_kind, w.rot_block, fmt=fmt, levels=levels)
    kc, kp = c.new_pools(fill=0)
    vc, vp = c.new_pools(fill=0)
    K, V, TS, TP, BT = dev(k), dev(v), dev(ts), dev(tp), dev(w.block_table)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kvq.quantize_append(c, K, V, TS, TP, BT, kc, kp, vc, vp, err=err)
    if which == "append":
        for _ in range(4):
            kvq.quantize_append(c, K, V, TS, TP, BT, kc, kp, vc, vp, err=err)
    else:
        del K, V
        q, lens = dev(w.queries()), dev(w.seq_lens)
        L = int(w.seq_lens.max())
        ws = torch.zeros(kvq.decode_workspace_bytes(c, w.S, w.Hq, L), dtype=torch.uint8,
                         device="cuda")
        for _ in range(4):
            kvq.paged_decode_attn(c, q, lens, L, BT, kc, kp, vc, vp, workspace=ws, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0, f"device error flags {int(err.item())}"
    print(f"profile case {which} done")


def _device_time_us(fn, n=20):
    """Median over 5 rounds of n back-to-back launches, CUDA events, in us."""
    for i in range(3):
        fn(i)
    torch.cuda.synchronize()
    ts = []
    for _ in range(5):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(n):
            fn(i)
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) / n)
    return float(np.median(ts)) * 1e3


def _device_kv(w, T, gen, device):
    """K and V [T][H][d] binary16 of a workload's shape and value structure
    (N(0,1) draws times its per-(head, channel) multipliers), drawn on the
    device so that the large workloads need no host-side generation. Timing
    only: the parity tests use the seeded host draws."""
    mult = (torch.ones((w.H, w.d)) if w.channel_mult is None
            else torch.from_numpy(w.channel_mult)).to(device)
    out = []
    for _ in range(2):
        x = torch.empty((T, w.H, w.d), dtype=torch.float16, device=device)
        for t0 in range(0, T, 1 << 16):
            t1 = min(T, t0 + (1 << 16))
            x[t0:t1] = (torch.randn((t1 - t0, w.H, w.d), generator=gen, device=device)
                        * mult).half()
        out.append(x)
    return out


def _all_tokens(w):
    """(token_seq, token_pos) of every cached token, sequence-major."""
    lens = w.seq_lens.astype(np.int64)
    ts = np.repeat(np.arange(w.S, dtype=np.int32), lens)
    tp = np.concatenate([np.arange(n, dtype=np.int32) for n in lens])
    return ts, tp


def _rate(nbytes, us, peak):
    gbs = nbytes / us / 1e3
    return {"us": us, "gbs": gbs, "frac": gbs / peak, "frac_nominal": gbs / NOMINAL_HBM_GBS,
            "bytes": int(nbytes)}


def workload_records(device, seed=0):
    """The other workloads on one GPU, each timed by CUDA events (median of 5
    rounds of back-to-back launches; every launch reads more than the 126 MB
    L2, or alternates between two cache replicas that together do):

    * long-context 70B-shaped decode (8 x 32768 tokens, GQA 8, page 32) over
      INT4 pages with Hadamard b 128, over INT4 pages without rotation, and
      over binary16 pages (the full-precision baseline);
    * the bulk prefill append of one layer (65536 tokens x 8 KV heads) per
      Hadamard block size and without rotation, with the reconstruction MSE
      of the INT4 cache (GPU dequantization, un-rotated, against the input);
    * the ragged head_dim-256 workload (128 sequences, lengths 512-16384):
      one fused decode step (append + attention) with Hadamard b 256 and with
      the quaternion rotation;
    * the cache formats against INT4 on the Llama-shaped layer -- microscaled
      FP4 (E2M1 codes, UE8M0 block scales, decode QK on the block-scaled
      tensor-core MMA), 3- and 2-bit codes and the calibrated level table
      (decode QK on the integer tensor-core MMA): bulk append, fused decode
      step, reconstruction MSE; FP4 also on the long-context decode.
    """
    from bit_rotated_kv_block_b200 import kvq, workloads
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(device)
    peak, _ = measured_peaks()
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    res = {}

    # ---- long-context 70B-shaped decode
    w = workloads.long70b(seed=seed)
    ts, tp = _all_tokens(w)
    K, V = _device_kv(w, len(ts), gen, device)
    TS, TP, BT = dev(ts), dev(tp), dev(w.block_table)
    q, lens, L = dev(w.queries()), dev(w.seq_lens), int(w.seq_lens.max())
    out = torch.empty((w.S, w.Hq, w.d), dtype=torch.float32, device=device)
    n_th = int(w.seq_lens.sum()) * w.H
    rec = {"workload": "8 seqs x 32768 tokens, 8 KV heads, 64 q heads, d 128, page 32"}
    for rot, blk, name, fmt in ((workloads.ROT_HADAMARD, 128, "int4_hadamard128", kvq.FMT_INT4),
                                (workloads.ROT_NONE, 0, "int4_no_rotation", kvq.FMT_INT4),
                                (workloads.ROT_HADAMARD, 128, "mxfp4_hadamard128",
                                 kvq.FMT_MXFP4)):
        reps = []
        for _ in range(2):
            c = kvq.Cache(w.d, w.H, w.P, w.NP, rot, blk, device=device, fmt=fmt)
            kc, kp = c.new_pools(device=device, fill=0)
            vc, vp = c.new_pools(device=device, fill=0)
            kvq.quantize_append(c, K, V, TS, TP, BT, kc, kp, vc, vp)
            reps.append((c, kc, kp, vc, vp))
        ws = torch.zeros(kvq.decode_workspace_bytes(reps[0][0], w.S, w.Hq, L), dtype=torch.uint8,
                         device=device)
        t = _device_time_us(lambda i: kvq.paged_decode_attn(
            reps[i % 2][0], q, lens, L, BT, *reps[i % 2][1:], out=out, workspace=ws))
        rec[name] = _rate(n_th * BYTES_PER_TOKEN_HEAD, t, peak)
        del reps, ws
    page = BT[TS.long(), (TP // w.P).long()].long()
    slot = (TP % w.P).long()
    reps = []
    for _ in range(2):
        kp16 = torch.zeros((w.NP, w.H, w.P, w.d), dtype=torch.float16, device=device)
        vp16 = torch.zeros_like(kp16)
        kp16[page, :, slot, :] = K
        vp16[page, :, slot, :] = V
        reps.append((kp16, vp16))
    c16 = kvq.Cache(w.d, w.H, w.P, w.NP, workloads.ROT_NONE, 0, device=device)
    ws = torch.zeros(kvq.decode_fp16_workspace_bytes(c16, w.S, w.Hq, L), dtype=torch.uint8,
                     device=device)
    t = _device_time_us(lambda i: kvq.paged_decode_attn_fp16(
        c16, q, lens, L, BT, reps[i % 2][0], reps[i % 2][1], out=out, workspace=ws))
    rec["fp16_baseline"] = _rate(n_th * 512, t, peak)
    rec["rotation_overhead"] = rec["int4_hadamard128"]["us"] / rec["int4_no_rotation"]["us"] - 1
    rec["speedup_vs_fp16"] = rec["fp16_baseline"]["us"] / rec["int4_hadamard128"]["us"]
    res["long70b_decode"] = rec
    del reps, ws, K, V, page, slot, TS, TP
    torch.cuda.empty_cache()

    # ---- prefill sweep: one layer per Hadamard block size, then the other
    # rotation kinds (quaternion full, fast and matrix maps, randomised-sign
    # b 64)
    sweep = {"workload": "65536 tokens x 8 KV heads x d 128 per layer, page 16"}
    variants = [(workloads.ROT_HADAMARD, b, "hadamard%d" % b) for b in (16, 32, 64, 128)]
    variants += [(workloads.ROT_NONE, 0, "no_rotation"),
                 (workloads.ROT_QUAT, 0, "quaternion"),
                 (workloads.ROT_QUAT_FAST, 0, "quaternion_fast"),
                 (workloads.ROT_QUAT_MAT, 0, "quaternion_matrix"),
                 (workloads.ROT_HADAMARD_SIGNED, 64, "hadamard64_signed")]
    for kind, blk, name in variants:
        w = workloads.prefill(seed=seed, rot_block=blk)
        ts, tp = _all_tokens(w)
        K, V = _device_kv(w, len(ts), gen, device)
        TS, TP, BT = dev(ts), dev(tp), dev(w.block_table)
        table = None
        if kind in (workloads.ROT_QUAT, workloads.ROT_QUAT_FAST, workloads.ROT_QUAT_MAT):
            table = workloads.random_quaternions(seed, w.d)
        elif kind == workloads.ROT_HADAMARD_SIGNED:
            table = workloads.random_signs(seed, w.d)
        c = kvq.Cache(w.d, w.H, w.P, w.NP, kind, blk, table, device=device)
        kc, kp = c.new_pools(device=device, fill=0)
        vc, vp = c.new_pools(device=device, fill=0)
        t = _device_time_us(lambda i: kvq.quantize_append(c, K, V, TS, TP, BT, kc, kp, vc, vp),
                            n=10)
        r = _rate(len(ts) * w.H * APPEND_BYTES_PER_TOKEN_HEAD, t, peak)
        lens = dev(np.full(w.S, int(w.seq_lens[0]), np.int32))
        Lmax = int(w.seq_lens[0])
        mse = 0.0
        for codes, params, src in ((kc, kp, K), (vc, vp, V)):
            xh = kvq.dequantize_pages(c, lens, Lmax, BT, codes, params, unrotate=True)
            x = src.view(w.S, Lmax, w.H, w.d).double()
            mse += float(((xh.double() - x) ** 2).mean()) / 2
            del xh, x
        r["mse"] = mse
        sweep[name] = r
        del K, V, kc, kp, vc, vp
        torch.cuda.empty_cache()
    for name in sweep:
        if name not in ("workload", "no_rotation"):
            sweep[name]["rotation_overhead"] = sweep[name]["us"] / sweep["no_rotation"]["us"] - 1
    res["prefill_append_sweep"] = sweep

    # ---- ragged head_dim 256: one fused decode step over the whole batch
    rec = {"workload": "128 seqs, lengths U[512, 16384], 4 KV heads, 16 q heads, d 256, page 16"}
    for rot, name in ((workloads.ROT_HADAMARD, "hadamard256"), (workloads.ROT_QUAT, "quaternion")):
        w = workloads.ragged256(seed=seed, rot_kind=rot)
        ts, tp = _all_tokens(w)
        K, V = _device_kv(w, len(ts), gen, device)
        c = kvq.Cache(w.d, w.H, w.P, w.NP, w.rot_kind, w.rot_block, w.quat, device=device)
        kc, kp = c.new_pools(device=device, fill=0)
        vc, vp = c.new_pools(device=device, fill=0)
        BT = dev(w.block_table)
        kvq.quantize_append(c, K, V, dev(ts), dev(tp), BT, kc, kp, vc, vp)
        del K, V
        kn = torch.randn((w.S, w.H, w.d), generator=gen, device=device).half()
        vn = torch.randn((w.S, w.H, w.d), generator=gen, device=device).half()
        lens_np = (w.seq_lens + 1).astype(np.int32)
        lens, L = dev(lens_np), int(lens_np.max())
        q = dev(w.queries())
        out = torch.empty((w.S, w.Hq, w.d), dtype=torch.float32, device=device)
        ws = torch.zeros(kvq.decode_workspace_bytes(c, w.S, w.Hq, L), dtype=torch.uint8,
                         device=device)
        t = _device_time_us(lambda i: kvq.decode_step(c, q, kn, vn, lens, L, BT, kc, kp, vc, vp,
                                                      out=out, workspace=ws))
        n_tok = int(lens_np.sum())
        r = _rate(n_tok * w.H * (w.d + 8), t, peak)
        r["kv_tokens"] = n_tok
        rec["step_" + name] = r
        del kc, kp, vc, vp, ws
        torch.cuda.empty_cache()
    res["ragged256_step"] = rec

    # ---- the cache formats on the Llama-shaped layer (INT4, microscaled FP4,
    # 3- and 2-bit codes, the calibrated level table): bulk append, fused
    # decode step, reconstruction MSE; bytes per token-head from each
    # format's row size
    from bit_rotated_kv_block_b200 import calibrate
    w = workloads.llama8b(seed=seed)
    levels = calibrate.calibrate_levels(
        np.random.default_rng([seed, 77]).standard_normal((4000, w.d)), w.rot_block)
    ts, tp = _all_tokens(w)
    K, V = _device_kv(w, len(ts), gen, device)
    TS, TP, BT = dev(ts), dev(tp), dev(w.block_table)
    rec = {"workload": "32 seqs x 4096 tokens + 1, 8 KV heads, 32 q heads, d 128, page 16, "
                       "Hadamard b 64"}
    Lc = int(w.seq_lens[0])
    lens_c = dev(np.full(w.S, Lc, np.int32))
    for fmt, name in ((kvq.FMT_INT4, "int4"), (kvq.FMT_MXFP4, "mxfp4"), (kvq.FMT_INT3, "int3"),
                      (kvq.FMT_INT2, "int2"), (kvq.FMT_LUT4, "lut4_calibrated")):
        c = kvq.Cache(w.d, w.H, w.P, w.NP, w.rot_kind, w.rot_block, device=device, fmt=fmt,
                      levels=levels if fmt == kvq.FMT_LUT4 else None)
        row_b = 2 * (c.code_row_bytes() + 4)  # K and V codes + params per token-head
        kc, kp = c.new_pools(device=device, fill=0)
        vc, vp = c.new_pools(device=device, fill=0)
        t = _device_time_us(lambda i: kvq.quantize_append(c, K, V, TS, TP, BT, kc, kp, vc, vp),
                            n=10)
        r = {"append": _rate(len(ts) * w.H * (4 * w.d + row_b), t, peak),
             "bytes_per_token_head": row_b}
        mse = 0.0
        for codes, params, src in ((kc, kp, K), (vc, vp, V)):
            xh = kvq.dequantize_pages(c, lens_c, Lc, BT, codes, params, unrotate=True)
            x = src.view(w.S, Lc, w.H, w.d).double()
            mse += float(((xh.double() - x) ** 2).mean()) / 2
            del xh, x
        r["mse"] = mse
        kn = torch.randn((w.S, w.H, w.d), generator=gen, device=device).half()
        vn = torch.randn((w.S, w.H, w.d), generator=gen, device=device).half()
        lens_np = (w.seq_lens + 1).astype(np.int32)
        lens, L = dev(lens_np), int(lens_np.max())
        q = dev(w.queries())
        out = torch.empty((w.S, w.Hq, w.d), dtype=torch.float32, device=device)
        ws = torch.zeros(kvq.decode_workspace_bytes(c, w.S, w.Hq, L), dtype=torch.uint8,
                         device=device)
        t = _device_time_us(lambda i: kvq.decode_step(c, q, kn, vn, lens, L, BT, kc, kp, vc, vp,
                                                      out=out, workspace=ws))
        r["step"] = _rate(int(lens_np.sum()) * w.H * row_b, t, peak)
        rec[name] = r
        del kc, kp, vc, vp, ws
        torch.cuda.empty_cache()
    del K, V
    rec["levels"] = [float(x) for x in levels]
    res["formats_llama8b"] = rec
    res["peak_gbs"] = peak
    res["nominal_gbs"] = NOMINAL_HBM_GBS
    return res


def compare():
    print(json.dumps({"mode": "compare", **workload_records(torch.device("cuda", 0))}), flush=True)


def main():
    args = parse()
    if args.compare:
        compare()
        return
    if args.profile_case:
        profile_case(args.profile_case, args.profile_block, args.profile_workload)
        return
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            line = run_reference(args, world, rank)
            if line is not None:
                print(json.dumps(line), flush=True)
            return
        res = run_ours(args, world, rank, local)
        if res is None:
            return
        line, w = res
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, args.cpu_budget)
        print(json.dumps(line), flush=True)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
