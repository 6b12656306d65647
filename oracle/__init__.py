"""Plain CPU oracle for the rotated token-wise INT4 paged KV cache.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / reference leg may import this package. It shares
no code with the CUDA library in ``bit_rotated_kv_block_b200``; both sides are
fed the same seeded inputs from ``bit_rotated_kv_block_b200.workloads``, which
holds none of the method's arithmetic.

The arithmetic lives in ``kvq_oracle.cpp`` (plain loops, IEEE binary32 in the
order written for the quantize path, double precision for attention); this
module only marshals numpy arrays. Method sources, by page title and section:

* "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM
  Serving" -- Summary, Method: token-wise INT4 with block-diagonal Hadamard
  rotation, fused into paged KV-cache layouts.
* "UltraQuant: 4-bit KV caching for long agents" -- how the method works:
  Walsh-Hadamard rotation spreads outliers across channels.
* "IsoQuant: Hardware-Aligned SO(4) Isoclinic Rotations for LLM KV Cache
  Compression" -- Abstract: T(v) = qL v conj(qR) per 4-D block.

Every function here is pinned by ``tests/test_oracle_*.py`` against
closed forms, textbook identities, library routines and brute force. The
pages print no worked example or table that this path reproduces, so none of
those pins is a number taken from them.
"""

import ctypes
import os

import numpy as np

from . import build as _build

ROT_NONE, ROT_HADAMARD, ROT_QUAT, ROT_QUAT_FAST, ROT_HADAMARD_SIGNED, ROT_QUAT_MAT = 0, 1, 2, 3, 4, 5
FMT_INT4, FMT_MXFP4, FMT_INT2, FMT_INT3, FMT_LUT4 = 0, 1, 2, 3, 4
RN, RD, RU = 0, 1, 2
ERR_PAGE, ERR_POS, ERR_SEQ, ERR_LEN = 1, 2, 4, 8

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        sig = {
            "orc_half_to_double": (dbl, [ctypes.c_uint16]),
            "orc_float_to_half": (ctypes.c_uint16, [ctypes.c_float, i32]),
            "orc_hadamard_scale": (ctypes.c_float, [i32]),
            "orc_sub_ru": (ctypes.c_float, [ctypes.c_float, ctypes.c_float]),
            "orc_div_ru": (ctypes.c_float, [ctypes.c_float, ctypes.c_float]),
            "orc_hamilton_f32": (None, [P, P, P]),
            "orc_quat_matrix_f32": (None, [P, P]),
            "orc_float_to_half_array": (None, [P, i64, i32, P]),
            "orc_double_to_half_array": (None, [P, i64, i32, P]),
            "orc_half_to_double_array": (None, [P, i64, P]),
            "orc_rotate_rows_f32": (None, [P, i64, i32, i32, i32, P]),
            "orc_rotate_rows_f64": (None, [P, i64, i32, i32, i32, P]),
            "orc_unrotate_rows_f64": (None, [P, i64, i32, i32, i32, P]),
            "orc_fwht_unscaled": (None, [P, i32]),
            "orc_quantize_rows": (None, [P, i64, i32, P, P, P]),
            "orc_quantize_append": (None, [i32, i32, i32, i32, i32, i32, P, i32, P, P, i64,
                                           P, P, i32, P, i32, P, P, P, P, P, i32, i32, P, P]),
            "orc_dequantize_pages": (None, [i32, i32, i32, i32, i32, i32, P, i32, P, i32, P,
                                            i32, P, P, i32, i32, P, i32, P, P]),
            "orc_paged_decode_attn": (None, [i32, i32, i32, i32, i32, i32, P, i32, i32, P, P,
                                             i32, P, i32, dbl, P, P, P, P, P, i32, i32, P,
                                             P, P]),
            "orc_quantize_rows_fmt": (None, [P, i64, i32, i32, P, P, P, P]),
            "orc_unpack_codes_rows": (None, [P, i64, i32, i32, P]),
            "orc_mx_exponent": (i32, [ctypes.c_float, i32]),
            "orc_e2m1_encode": (i32, [dbl]),
            "orc_e2m1_value": (dbl, [i32]),
            "orc_e4m3_encode": (i32, [dbl]),
            "orc_e4m3_value": (dbl, [i32]),
            "orc_mxfp4_quantize_row": (None, [P, i32, P, P]),
            "orc_mxfp8_row_values": (None, [P, i32, P]),
            "orc_rope_row_f32": (None, [P, i32, P]),
            "orc_paged_decode_attn_fp16": (None, [i32, i32, i32, i32, i32, i32, P, P, i32, P,
                                                  i32, dbl, P, P, P, P]),
            "orc_num_threads": (i32, []),
            "orc_set_num_threads": (None, [i32]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _p(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _quat(quat):
    return None if quat is None else _c(quat, np.float32)


# --- binary16 -------------------------------------------------------------

def float_to_half_bits(x, mode=RN):
    """binary32 -> binary16 bits (uint16) with RN / RD / RU rounding."""
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().orc_float_to_half_array(_p(x), x.size, mode, _p(out))
    return out


def double_to_half_bits(x, mode=RN):
    x = _c(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    lib().orc_double_to_half_array(_p(x), x.size, mode, _p(out))
    return out


def half_bits_to_double(h):
    h = _c(h, np.uint16)
    out = np.empty(h.shape, np.float64)
    lib().orc_half_to_double_array(_p(h), h.size, _p(out))
    return out


# --- rotary position embedding (optional, in front of the rotation) --------

def rope_rows_f32(x, cs):
    """Turns rows x (float32 [n][d]) by the RoPE table rows cs (float32
    [n][d/2][2] of (cos, sin), one per row): binary32, products and the
    difference / sum rounded separately."""
    x = _c(x, np.float32).copy()
    cs = _c(cs, np.float32).reshape(x.shape[0], -1)
    for i in range(x.shape[0]):
        lib().orc_rope_row_f32(x[i].ctypes.data, x.shape[1], cs[i].ctypes.data)
    return x


# --- rotation ---------------------------------------------------------------

def hadamard_scale(b):
    return lib().orc_hadamard_scale(int(b))


def sub_ru(a, b):
    """binary32 a - b rounded toward +inf."""
    return np.float32(lib().orc_sub_ru(float(a), float(b)))


def div_ru(a, b):
    """binary32 a / b rounded toward +inf."""
    return np.float32(lib().orc_div_ru(float(a), float(b)))


def fwht_unscaled(x):
    """Unscaled fast Walsh-Hadamard transform of one block (binary32)."""
    x = _c(x, np.float32).copy()
    lib().orc_fwht_unscaled(_p(x), x.size)
    return x


def hamilton(a, b):
    a, b = _c(a, np.float32), _c(b, np.float32)
    out = np.empty(4, np.float32)
    lib().orc_hamilton_f32(_p(a), _p(b), _p(out))
    return out


def quat_matrix(q8):
    """The binary32 4x4 matrix of v -> qL v conj(qR) for one table entry
    (qL, qR) as the matrix-form rotation builds it."""
    q8 = _c(q8, np.float32).reshape(8)
    out = np.empty(16, np.float32)
    lib().orc_quat_matrix_f32(_p(q8), _p(out))
    return out.reshape(4, 4)


def rotate_f32(x, kind, block=0, quat=None):
    """Forward rotation of rows (last axis = d) in the binary32 order of the
    quantize path."""
    x = _c(x, np.float32).copy()
    d = x.shape[-1]
    q = _quat(quat)
    lib().orc_rotate_rows_f32(_p(x), x.size // d, d, kind, block, _p(q))
    return x


def rotate_f64(x, kind, block=0, quat=None):
    x = _c(x, np.float64).copy()
    d = x.shape[-1]
    q = _quat(quat)
    lib().orc_rotate_rows_f64(_p(x), x.size // d, d, kind, block, _p(q))
    return x


def unrotate_f64(x, kind, block=0, quat=None):
    x = _c(x, np.float64).copy()
    d = x.shape[-1]
    q = _quat(quat)
    lib().orc_unrotate_rows_f64(_p(x), x.size // d, d, kind, block, _p(q))
    return x


# --- microscaled FP4 / FP8 -------------------------------------------------------

def mx_exponent(amax, emax):
    return lib().orc_mx_exponent(float(amax), int(emax))


def e2m1_encode(t):
    return lib().orc_e2m1_encode(float(t))


def e2m1_value(code):
    return lib().orc_e2m1_value(int(code))


def e4m3_encode(t):
    return lib().orc_e4m3_encode(float(t))


def e4m3_value(code):
    return lib().orc_e4m3_value(int(code))


def mxfp4_quantize_rows(y):
    """Rotated binary32 rows [..., d] -> (E2M1 codes uint8 [..., d/2], UE8M0
    scales uint8 [..., d/32])."""
    y = _c(y, np.float32)
    d = y.shape[-1]
    flat = y.reshape(-1, d)
    codes = np.empty((flat.shape[0], d // 2), np.uint8)
    scales = np.empty((flat.shape[0], d // 32), np.uint8)
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        cr, sr = codes[r], scales[r]
        lib().orc_mxfp4_quantize_row(_p(row), d, _p(cr), _p(sr))
    return codes.reshape(y.shape[:-1] + (d // 2,)), scales.reshape(y.shape[:-1] + (d // 32,))


def mxfp8_values(y):
    """Rotated binary32 rows [..., d] -> their MX E4M3 values (float64)."""
    y = _c(y, np.float32)
    d = y.shape[-1]
    flat = y.reshape(-1, d)
    out = np.empty(flat.shape, np.float64)
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        o = out[r]
        lib().orc_mxfp8_row_values(_p(row), d, _p(o))
    return out.reshape(y.shape)


def quantize_rows_fmt(y, fmt, levels=None):
    """Rotated binary32 rows [..., d] -> (packed codes uint8 [..., d*bits/8],
    s16 bits, m16 bits) for FMT_INT2 / FMT_INT3 / FMT_INT4 / FMT_LUT4."""
    y = _c(y, np.float32)
    d = y.shape[-1]
    rows = y.size // d
    bits = {FMT_INT2: 2, FMT_INT3: 3}.get(fmt, 4)
    codes = np.empty(y.shape[:-1] + (d * bits // 8,), np.uint8)
    s16 = np.empty(y.shape[:-1], np.uint16)
    m16 = np.empty(y.shape[:-1], np.uint16)
    lv = None if levels is None else _c(levels, np.float32)
    lib().orc_quantize_rows_fmt(_p(y), rows, d, int(fmt), _p(lv), _p(codes), _p(s16), _p(m16))
    return codes, s16, m16


def unpack_codes_bits(codes, d, bits):
    """Packed rows [..., d*bits/8] -> integer codes int32 [..., d]."""
    codes = _c(codes, np.uint8)
    rows = codes.size // (d * bits // 8)
    out = np.empty(codes.shape[:-1] + (d,), np.int32)
    lib().orc_unpack_codes_rows(_p(codes), rows, d, bits, _p(out))
    return out


# --- quantizer ----------------------------------------------------------------

def quantize_rows(y):
    """Token-wise INT4 of already-rotated binary32 rows.

    Returns (codes uint8 [..., d/2], s16 bits uint16 [...], m16 bits uint16 [...]).
    """
    y = _c(y, np.float32)
    d = y.shape[-1]
    rows = y.size // d
    codes = np.empty(y.shape[:-1] + (d // 2,), np.uint8)
    s16 = np.empty(y.shape[:-1], np.uint16)
    m16 = np.empty(y.shape[:-1], np.uint16)
    lib().orc_quantize_rows(_p(y), rows, d, _p(codes), _p(s16), _p(m16))
    return codes, s16, m16


def unpack_codes(codes):
    codes = np.asarray(codes, np.uint8)
    out = np.empty(codes.shape[:-1] + (codes.shape[-1] * 2,), np.int32)
    out[..., 0::2] = codes & 0xF
    out[..., 1::2] = codes >> 4
    return out


def dequantize_rows(codes, s16, m16):
    """x = c * s16 + m16 in double (exact)."""
    c = unpack_codes(codes).astype(np.float64)
    s = half_bits_to_double(s16)[..., None]
    m = half_bits_to_double(m16)[..., None]
    return c * s + m


# --- cache-level operations (same contract as the library's entry points) ----

class Cache:
    """Geometry of one paged cache (head_dim d, KV heads H, page size P,
    pool size NP, rotation kind / block / quaternion table) and its format:
    FMT_INT4 (token-wise INT4, params (s16, m16)) or FMT_MXFP4 (E2M1 codes,
    one UE8M0 byte per 32 channels, a 4-byte params row)."""

    def __init__(self, d, H, P, NP, rot_kind, rot_block=0, quat=None, rope=None, fmt=FMT_INT4,
                 levels=None):
        self.fmt = int(fmt)
        # the LUT4 format's 16 levels (float32, binary16-exact, on the 1/16 grid)
        self.levels = None if levels is None else _c(levels, np.float32).reshape(16)
        assert (self.levels is not None) == (self.fmt == FMT_LUT4)
        self.d, self.H, self.P, self.NP = int(d), int(H), int(P), int(NP)
        self.rot_kind, self.rot_block = int(rot_kind), int(rot_block)
        self.quat = _quat(quat)
        # optional RoPE table float32 [max_pos][d/2][2] of (cos, sin)
        self.rope = None if rope is None else _c(rope, np.float32).reshape(-1, self.d)
        self.rope_max_pos = 0 if rope is None else self.rope.shape[0]

    def code_row_bytes(self):
        return self.d * {FMT_INT2: 2, FMT_INT3: 3}.get(self.fmt, 4) // 8

    def alloc_pools(self, fill=0):
        codes = np.full((self.NP, self.H, self.P, self.code_row_bytes()), fill, np.uint8)
        if self.fmt == FMT_MXFP4:
            params = np.full((self.NP, self.H, self.P, max(4, self.d // 32)), fill, np.uint8)
        else:
            params = np.full((self.NP, self.H, self.P, 2), (fill << 8) | fill, np.uint16)
        return codes, params

    def params_array(self, params):
        """A params pool as the C code reads it (bytes for MX FP4)."""
        return _c(params, np.uint8 if self.fmt == FMT_MXFP4 else np.uint16)


def quantize_append(cache, k, v, token_seq, token_pos, block_table, k_codes, k_params,
                    v_codes, v_params, tok_stride=None, num_seqs=None):
    """Rotate, quantize, pack and scatter T tokens of K and V (binary16 bits,
    [T][H][d] with token stride ``tok_stride`` elements) into the pools, in
    place. Returns the OR of error flags."""
    # converted copies are bound to names so they outlive the C call
    k, v = _c(k, np.uint16), _c(v, np.uint16)
    ts, tp = _c(token_seq, np.int32), _c(token_pos, np.int32)
    T = len(ts)
    if tok_stride is None:
        tok_stride = cache.H * cache.d
    bt = _c(block_table, np.int32)
    if num_seqs is None:
        num_seqs = bt.shape[0]
    err = np.zeros(1, np.int32)
    for a in (k_codes, k_params, v_codes, v_params):
        assert a.flags.c_contiguous
    lib().orc_quantize_append(cache.d, cache.H, cache.P, cache.NP, cache.rot_kind,
                              cache.rot_block, _p(cache.quat), T, _p(k), _p(v), tok_stride,
                              _p(ts), _p(tp), num_seqs, _p(bt), bt.shape[1], _p(k_codes),
                              _p(k_params), _p(v_codes), _p(v_params), _p(cache.rope),
                              cache.rope_max_pos, cache.fmt, _p(cache.levels), _p(err))
    return int(err[0])


def dequantize_pages(cache, seq_lens, max_seq_len, block_table, codes, params, unrotate,
                     out_fp32=True, out=None):
    bt = _c(block_table, np.int32)
    lens = _c(seq_lens, np.int32)
    codes, params = _c(codes, np.uint8), cache.params_array(params)
    S = bt.shape[0]
    shape = (S, max_seq_len, cache.H, cache.d)
    if out is None:
        out = np.zeros(shape, np.float32 if out_fp32 else np.uint16)
    err = np.zeros(1, np.int32)
    lib().orc_dequantize_pages(cache.d, cache.H, cache.P, cache.NP, cache.rot_kind,
                               cache.rot_block, _p(cache.quat), S, _p(lens), max_seq_len, _p(bt),
                               bt.shape[1], _p(codes), _p(params), int(bool(unrotate)),
                               int(bool(out_fp32)), _p(out), cache.fmt, _p(cache.levels),
                               _p(err))
    return out, int(err[0])


def paged_decode_attn(cache, q, seq_lens, max_seq_len, block_table, sm_scale, k_codes,
                      k_params, v_codes, v_params):
    """Decode attention in double precision; q is binary16 bits [S][Hq][d].
    Returns (out float64 [S][Hq][d], error flags)."""
    q = _c(q, np.uint16)
    S, Hq, d = q.shape
    bt = _c(block_table, np.int32)
    lens = _c(seq_lens, np.int32)
    kc, kp = _c(k_codes, np.uint8), cache.params_array(k_params)
    vc, vp = _c(v_codes, np.uint8), cache.params_array(v_params)
    out = np.empty((S, Hq, d), np.float64)
    err = np.zeros(1, np.int32)
    lib().orc_paged_decode_attn(cache.d, cache.H, cache.P, cache.NP, cache.rot_kind,
                                cache.rot_block, _p(cache.quat), S, Hq, _p(q), _p(lens),
                                max_seq_len, _p(bt), bt.shape[1], float(sm_scale), _p(kc),
                                _p(kp), _p(vc), _p(vp), _p(cache.rope), cache.rope_max_pos,
                                cache.fmt, _p(cache.levels), _p(out), _p(err))
    return out, int(err[0])


def paged_decode_attn_fp16(d, H, P, NP, q, seq_lens, max_seq_len, block_table, sm_scale,
                           k16, v16):
    q = _c(q, np.uint16)
    S, Hq, _ = q.shape
    bt = _c(block_table, np.int32)
    lens = _c(seq_lens, np.int32)
    k16, v16 = _c(k16, np.uint16), _c(v16, np.uint16)
    out = np.empty((S, Hq, d), np.float64)
    err = np.zeros(1, np.int32)
    lib().orc_paged_decode_attn_fp16(d, H, P, NP, S, Hq, _p(q), _p(lens), max_seq_len, _p(bt),
                                     bt.shape[1], float(sm_scale), _p(k16), _p(v16), _p(out),
                                     _p(err))
    return out, int(err[0])


def reconstruction_mse(x_orig_bits, x_hat):
    """Mean over elements of (x - xhat)^2 in double, x given as binary16 bits."""
    x = half_bits_to_double(x_orig_bits)
    return float(np.mean((x - np.asarray(x_hat, np.float64)) ** 2))


def num_threads():
    return lib().orc_num_threads()


def set_num_threads(n):
    lib().orc_set_num_threads(int(n))
