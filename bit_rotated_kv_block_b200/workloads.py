"""Seeded synthetic inputs for the rotated INT4 paged KV cache.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no rotation, no quantization, no attention), so both the
CUDA path and the CPU oracle can be fed from it without sharing any of the
computation they are compared on.

Every tensor has its own PCG64 stream, ``numpy.random.default_rng([seed,
workload_id, stream_id])``, so one tensor can be regenerated without the others.
The shapes and value distributions restate the five workloads the method is
measured on:

* ``tiny``       1 sequence x 256 tokens, 8 KV heads, head_dim 128, channels 3
                 and 77 scaled x20, Hadamard block 128, page 16, 32 query heads.
* ``llama8b``    32 sequences x 4096 tokens (+1 appended per decode step),
                 8 KV heads, 32 query heads, head_dim 128, 2% outlier channels
                 x U[10, 30] per KV head, a x10 first ("sink") token, Hadamard
                 block 64, page 16, shuffled block table.
* ``long70b``    8 sequences x 32768 tokens, 8 KV heads, 64 query heads,
                 head_dim 128, channels 3 and 77 scaled x20, Hadamard block 128,
                 page 32.
* ``prefill``    65536 new tokens (16 x 4096) per layer x 32 layers, 8 KV heads,
                 head_dim 128, page 16, one shuffled block table for all layers.
* ``ragged256``  128 sequences with lengths uniform in [512, 16384], 4 KV heads,
                 16 query heads, head_dim 256, per-(head, channel) scales
                 log-uniform in [0.1, 20], Hadamard block 256 or a seeded
                 quaternion table (64 blocks of 4 channels).

No public dataset is involved: the pages measure on model activations and a
multi-turn chat benchmark, neither of which exists here; these draws stand in
for them.
"""

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

ROT_NONE, ROT_HADAMARD, ROT_QUAT, ROT_QUAT_FAST, ROT_HADAMARD_SIGNED, ROT_QUAT_MAT = \
    0, 1, 2, 3, 4, 5

WORKLOAD_IDS = {"tiny": 1, "llama8b": 2, "long70b": 3, "prefill": 4, "ragged256": 5}

# stream ids: one per drawn tensor
S_K, S_V, S_Q, S_TABLE, S_OUTLIER_CH, S_OUTLIER_MULT, S_LENS, S_QUAT, S_SCALE, \
    S_STEP_K, S_STEP_V = range(1, 12)


def rng(seed: int, workload: str, stream: int, extra: int = 0) -> np.random.Generator:
    return np.random.default_rng([int(seed), WORKLOAD_IDS[workload], int(stream), int(extra)])


def normal_f16(g: np.random.Generator, shape, chunk: int = 1 << 24) -> np.ndarray:
    """Standard normal draws rounded to binary16 (numpy's nearest-even cast)."""
    out = np.empty(int(np.prod(shape)), np.float16)
    flat = out.reshape(-1)
    for i in range(0, flat.size, chunk):
        n = min(chunk, flat.size - i)
        flat[i:i + n] = g.standard_normal(n, dtype=np.float32)
    return out.reshape(shape)


def scaled_normal_f16(g: np.random.Generator, shape, channel_mult: np.ndarray,
                      chunk_tokens: int = 1 << 15) -> np.ndarray:
    """N(0,1) draws times a per-(head, channel) multiplier [H][d], then binary16.

    ``shape`` is [T][H][d]; the multiplication is done in binary32 before the
    cast, chunked over tokens to bound memory.
    """
    T, H, d = shape
    out = np.empty(shape, np.float16)
    mult = channel_mult.astype(np.float32)[None]
    for t0 in range(0, T, chunk_tokens):
        t1 = min(T, t0 + chunk_tokens)
        x = g.standard_normal((t1 - t0, H, d), dtype=np.float32)
        out[t0:t1] = x * mult
    return out


def unit_quaternions(g: np.random.Generator, nblocks: int) -> np.ndarray:
    """Table [nblocks][2][4] float32 of (qL, qR), each four standard normals
    divided by their norm in float64 and then rounded to float32."""
    x = g.standard_normal((nblocks, 2, 4))
    x = x / np.linalg.norm(x, axis=-1, keepdims=True)
    return x.astype(np.float32)


def shuffled_pages(g: np.random.Generator, num_pages: int) -> np.ndarray:
    return g.permutation(num_pages).astype(np.int32)


@dataclass
class Workload:
    name: str
    d: int
    H: int
    Hq: int
    P: int
    NP: int
    rot_kind: int
    rot_block: int
    seq_lens: np.ndarray                 # int32 [S]: cached tokens per sequence
    block_table: np.ndarray              # int32 [S][bt_stride]
    quat: Optional[np.ndarray] = None    # float32 [d/4][2][4]
    channel_mult: Optional[np.ndarray] = None  # float32 [H][d] (or None: all 1)
    sink_mult: float = 1.0               # multiplier on token 0 of each sequence
    seed: int = 0
    notes: dict = field(default_factory=dict)

    @property
    def S(self):
        return int(self.block_table.shape[0])

    @property
    def bt_stride(self):
        return int(self.block_table.shape[1])

    @property
    def max_seq_len(self):
        return int(self.seq_lens.max()) if self.seq_lens.size else 0

    # --- token streams ---------------------------------------------------

    def kv(self, stream_k: int, stream_v: int, T: int, extra: int = 0):
        """K and V [T][H][d] binary16 for one batch of T tokens."""
        mult = self.channel_mult
        if mult is None:
            mult = np.ones((self.H, self.d), np.float32)
        k = scaled_normal_f16(rng(self.seed, self.name, stream_k, extra), (T, self.H, self.d), mult)
        v = scaled_normal_f16(rng(self.seed, self.name, stream_v, extra), (T, self.H, self.d), mult)
        return k, v

    def prefill_tokens(self, seqs=None, layer: int = 0):
        """All cached tokens of the given sequences, sequence-major: returns
        (k, v, token_seq, token_pos). Token 0 of every sequence is multiplied
        by ``sink_mult``."""
        if seqs is None:
            seqs = range(self.S)
        seqs = list(seqs)
        lens = [int(self.seq_lens[s]) for s in seqs]
        T = int(sum(lens))
        k, v = self.kv(S_K, S_V, T, extra=layer)
        token_seq = np.concatenate([np.full(n, s, np.int32) for s, n in zip(seqs, lens)]) \
            if T else np.zeros(0, np.int32)
        token_pos = np.concatenate([np.arange(n, dtype=np.int32) for n in lens]) \
            if T else np.zeros(0, np.int32)
        if self.sink_mult != 1.0:
            first = token_pos == 0
            k[first] = (k[first].astype(np.float32) * self.sink_mult).astype(np.float16)
            v[first] = (v[first].astype(np.float32) * self.sink_mult).astype(np.float16)
        return k, v, token_seq, token_pos

    def step_tokens(self, step: int = 0):
        """One new token per sequence at position seq_lens[s] (a decode step)."""
        k, v = self.kv(S_STEP_K, S_STEP_V, self.S, extra=step)
        token_seq = np.arange(self.S, dtype=np.int32)
        token_pos = self.seq_lens.astype(np.int32).copy()
        return k, v, token_seq, token_pos

    def queries(self, step: int = 0):
        """Decode queries [S][Hq][d] binary16, N(0,1) without outliers."""
        return normal_f16(rng(self.seed, self.name, S_Q, step), (self.S, self.Hq, self.d))


def _table(g, S, pages_per_seq, NP):
    perm = shuffled_pages(g, NP)
    return perm[:S * pages_per_seq].reshape(S, pages_per_seq).copy()


def tiny(seed: int = 0) -> Workload:
    d, H, P, NP = 128, 8, 16, 16
    mult = np.ones((H, d), np.float32)
    mult[:, [3, 77]] = 20.0
    table = shuffled_pages(rng(seed, "tiny", S_TABLE), NP)[None, :]
    return Workload("tiny", d, H, 32, P, NP, ROT_HADAMARD, 128,
                    np.array([256], np.int32), table, channel_mult=mult, seed=seed)


def llama8b(seed: int = 0, S: int = 32, ctx: int = 4096, spare_pages: int = 64) -> Workload:
    """Cached context ``ctx`` per sequence; the block table has room for one
    more page so decode steps can append at position ``ctx``."""
    d, H, P = 128, 8, 16
    pages_per_seq = (ctx + 1 + P - 1) // P
    NP = S * pages_per_seq + spare_pages
    g_ch = rng(seed, "llama8b", S_OUTLIER_CH)
    g_m = rng(seed, "llama8b", S_OUTLIER_MULT)
    n_out = int(round(0.02 * d))
    mult = np.ones((H, d), np.float32)
    for h in range(H):
        ch = g_ch.choice(d, size=n_out, replace=False)
        mult[h, ch] = g_m.uniform(10.0, 30.0, size=n_out).astype(np.float32)
    table = _table(rng(seed, "llama8b", S_TABLE), S, pages_per_seq, NP)
    return Workload("llama8b", d, H, 32, P, NP, ROT_HADAMARD, 64,
                    np.full(S, ctx, np.int32), table, channel_mult=mult, sink_mult=10.0,
                    seed=seed)


def long70b(seed: int = 0, S: int = 8, ctx: int = 32768, rot_kind: int = ROT_HADAMARD) -> Workload:
    d, H, P = 128, 8, 32
    pages_per_seq = (ctx + P - 1) // P
    NP = S * pages_per_seq
    mult = np.ones((H, d), np.float32)
    mult[:, [3, 77]] = 20.0
    table = _table(rng(seed, "long70b", S_TABLE), S, pages_per_seq, NP)
    return Workload("long70b", d, H, 64, P, NP, rot_kind, 128 if rot_kind == ROT_HADAMARD else 0,
                    np.full(S, ctx, np.int32), table, channel_mult=mult, seed=seed)


def prefill(seed: int = 0, rot_block: int = 128, S: int = 16, ctx: int = 4096) -> Workload:
    """One layer's worth of the bulk prefill write (``prefill_tokens(layer=l)``
    draws layer l); ``rot_block`` 0 means no rotation."""
    d, H, P = 128, 8, 16
    pages_per_seq = ctx // P
    NP = S * pages_per_seq
    mult = np.ones((H, d), np.float32)
    mult[:, [3, 77]] = 20.0
    table = _table(rng(seed, "prefill", S_TABLE), S, pages_per_seq, NP)
    kind = ROT_HADAMARD if rot_block else ROT_NONE
    return Workload("prefill", d, H, 8, P, NP, kind, rot_block, np.full(S, ctx, np.int32),
                    table, channel_mult=mult, seed=seed)


def ragged256(seed: int = 0, S: int = 128, lo: int = 512, hi: int = 16384,
              rot_kind: int = ROT_HADAMARD) -> Workload:
    d, H, P = 256, 4, 16
    lens = rng(seed, "ragged256", S_LENS).integers(lo, hi + 1, size=S).astype(np.int32)
    # room for one appended token per sequence
    pages = [(int(n) + 1 + P - 1) // P for n in lens]
    bt_stride = max(pages)
    NP = int(sum(pages))
    perm = shuffled_pages(rng(seed, "ragged256", S_TABLE), NP)
    table = np.full((S, bt_stride), -1, np.int32)
    off = 0
    for s, n in enumerate(pages):
        table[s, :n] = perm[off:off + n]
        off += n
    g_sc = rng(seed, "ragged256", S_SCALE)
    mult = np.exp(g_sc.uniform(np.log(0.1), np.log(20.0), size=(H, d))).astype(np.float32)
    quat = unit_quaternions(rng(seed, "ragged256", S_QUAT), d // 4)
    return Workload("ragged256", d, H, 16, P, NP, rot_kind,
                    256 if rot_kind == ROT_HADAMARD else 0, lens, table,
                    quat=quat if rot_kind in (ROT_QUAT, ROT_QUAT_FAST, ROT_QUAT_MAT) else None,
                    channel_mult=mult, seed=seed)


def random_quaternions(seed: int, d: int) -> np.ndarray:
    """A seeded quaternion table for head_dim d (d/4 blocks)."""
    return unit_quaternions(np.random.default_rng([int(seed), 99, S_QUAT]), d // 4)


def rope_table(max_pos: int, d: int, base: float = 10000.0) -> np.ndarray:
    """Rotary-position table float32 [max_pos][d/2][2]: (cos, sin) of
    pos * base^(-2i/d) for channel pair i = (2i, 2i+1), evaluated in float64
    and rounded to float32 (the table a serving stack precomputes once and
    hands to the cache; an input here, like the quaternion table)."""
    inv = base ** (-np.arange(0, d, 2, dtype=np.float64) / d)
    ang = np.arange(max_pos, dtype=np.float64)[:, None] * inv[None, :]
    return np.stack([np.cos(ang), np.sin(ang)], axis=-1).astype(np.float32)


def random_signs(seed: int, d: int) -> np.ndarray:
    """A seeded sign table float32 [d] of +1 / -1 (randomised-sign Hadamard)."""
    g = np.random.default_rng([int(seed), 98, S_QUAT])
    return g.choice(np.array([-1.0, 1.0], np.float32), size=d).astype(np.float32)
