"""ctypes binding over ``libkvq.so`` (C ABI in ``include/kvq.h``).

Argument marshalling only: every step of the rotated INT4 KV path runs in the
library's CUDA kernels. Tensors are torch CUDA tensors (used for device memory
and streams); their data pointers and sizes cross the C boundary. If the
library is missing this module raises on first use -- there is no fallback.
"""

import ctypes
import math
import os

import torch

from . import build as _build

ROT_NONE, ROT_HADAMARD, ROT_QUAT, ROT_QUAT_FAST, ROT_HADAMARD_SIGNED, ROT_QUAT_MAT = \
    0, 1, 2, 3, 4, 5
FMT_INT4, FMT_MXFP4, FMT_INT2, FMT_INT3, FMT_LUT4 = 0, 1, 2, 3, 4
ERRF_PAGE, ERRF_POS, ERRF_SEQ, ERRF_LEN = 1, 2, 4, 8
STATUS = {0: "KVQ_OK", 1: "KVQ_ERR_INVALID_ARG", 2: "KVQ_ERR_UNSUPPORTED",
          3: "KVQ_ERR_MISALIGNED", 4: "KVQ_ERR_WORKSPACE", 5: "KVQ_ERR_CUDA"}

# every function the header declares, with its ctypes signature
_P, _I32, _I64, _F32, _SZ = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                            ctypes.c_size_t)
SIGNATURES = {
    "kvq_quantize_append": (ctypes.c_int, [_P, _I32, _P, _P, _I64, _P, _P, _I32, _P, _I32, _P, _P,
                                           _P, _P, _P, _P]),
    "kvq_decode_workspace_bytes": (_SZ, [_P, _I32, _I32, _I32]),
    "kvq_paged_decode_attn": (ctypes.c_int, [_P, _I32, _I32, _P, _P, _I32, _P, _I32, _F32, _P, _P,
                                             _P, _P, _P, _P, _SZ, _P, _P]),
    "kvq_dequantize_pages": (ctypes.c_int, [_P, _I32, _P, _I32, _P, _I32, _P, _P, _I32, _I32, _P,
                                            _P, _P]),
    "kvq_paged_decode_attn_noalloc": (ctypes.c_int, [_P, _I32, _I32, _P, _P, _I32, _P, _I32, _F32,
                                                     _P, _P, _P, _P, _P, _P, _P]),
    "kvq_decode_step": (ctypes.c_int, [_P, _I32, _I32, _P, _P, _P, _I64, _P, _I32, _P, _I32, _F32,
                                       _P, _P, _P, _P, _P, _P, _SZ, _P, _P]),
    "kvq_decode_fp16_workspace_bytes": (_SZ, [_P, _I32, _I32, _I32]),
    "kvq_paged_decode_attn_fp16": (ctypes.c_int, [_P, _I32, _I32, _P, _P, _I32, _P, _I32, _F32,
                                                  _P, _P, _P, _P, _SZ, _P, _P]),
    "kvq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "kvq_version": (ctypes.c_char_p, []),
}


class KvqError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")
        self.status = status


class CacheDesc(ctypes.Structure):
    """Mirror of ``kvq_cache_desc``."""
    _fields_ = [("head_dim", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("rot_kind", ctypes.c_int32), ("rot_block", ctypes.c_int32),
                ("quat", ctypes.c_void_p), ("rope", ctypes.c_void_p),
                ("rope_max_pos", ctypes.c_int32), ("format", ctypes.c_int32),
                ("levels", ctypes.c_void_p)]


_lib = None


def lib_path():
    return _build.LIB


def lib():
    """Loads libkvq.so (built in-tree by ``build.build()``); raises if absent."""
    global _lib
    if _lib is None:
        path = lib_path()
        if not os.path.exists(path):
            raise RuntimeError(f"libkvq.so not built at {path}: run "
                               "bit_rotated_kv_block_b200.build.build() first")
        L = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn, status):
    if status != 0:
        raise KvqError(fn, status)


class Cache:
    """Geometry of one paged INT4 cache plus the device quaternion table
    (kept alive here because the descriptor points at it)."""

    def __init__(self, head_dim, num_kv_heads, page_size, num_pages, rot_kind=ROT_HADAMARD,
                 rot_block=0, quat=None, device="cuda", rope=None, fmt=FMT_INT4, levels=None):
        """``rope``: optional RoPE table float32 [max_pos][d/2][2] of (cos, sin);
        ``fmt``: a kvq_format; ``levels``: the 16-entry table of FMT_LUT4."""
        self.fmt = fmt
        self.levels = None
        if levels is not None:
            self.levels = torch.as_tensor(levels, dtype=torch.float32).contiguous().to(device)
        self.d, self.H, self.P, self.NP = head_dim, num_kv_heads, page_size, num_pages
        self.rot_kind, self.rot_block = rot_kind, rot_block
        self.quat = None  # the rotation's table: quaternions, or signs
        if rot_kind in (ROT_QUAT, ROT_QUAT_FAST, ROT_HADAMARD_SIGNED, ROT_QUAT_MAT):
            self.quat = torch.as_tensor(quat, dtype=torch.float32).contiguous().to(device)
        self.rope = None
        if rope is not None:
            self.rope = torch.as_tensor(rope, dtype=torch.float32).contiguous().to(device)
        self.desc = CacheDesc(head_dim, num_kv_heads, page_size, num_pages, rot_kind, rot_block,
                              None if self.quat is None else self.quat.data_ptr(),
                              None if self.rope is None else self.rope.data_ptr(),
                              0 if self.rope is None else int(self.rope.shape[0]), fmt,
                              None if self.levels is None else self.levels.data_ptr())

    def code_row_bytes(self):
        return self.d * {FMT_INT2: 2, FMT_INT3: 3}.get(self.fmt, 4) // 8

    def new_pools(self, device="cuda", fill=None):
        """(codes uint8 [NP][H][P][d * bits / 8], params int32 [NP][H][P]) for one
        of K / V; each params word is the binary16 pair (scale, minimum), scale in
        the low half (MX FP4: the four block-scale bytes)."""
        codes = torch.empty((self.NP, self.H, self.P, self.code_row_bytes()), dtype=torch.uint8,
                            device=device)
        params = torch.empty((self.NP, self.H, self.P), dtype=torch.int32, device=device)
        if fill is not None:
            codes.fill_(fill)
            params.fill_(int.from_bytes(bytes([fill] * 4), "little", signed=True))
        return codes, params


def quantize_append(cache, k, v, token_seq, token_pos, block_table, k_codes, k_params, v_codes,
                    v_params, err=None, stream=None, tok_stride=None):
    """k, v: float16 CUDA [T][H][d] (token stride ``tok_stride`` elements)."""
    T = int(token_seq.numel())
    if tok_stride is None:
        tok_stride = k.stride(0)
    st = lib().kvq_quantize_append(ctypes.byref(cache.desc), T, _ptr(k), _ptr(v), int(tok_stride),
                                   _ptr(token_seq), _ptr(token_pos), int(block_table.shape[0]),
                                   _ptr(block_table), int(block_table.shape[1]), _ptr(k_codes),
                                   _ptr(k_params), _ptr(v_codes), _ptr(v_params), _ptr(err),
                                   _stream(stream))
    _check("kvq_quantize_append", st)


def decode_workspace_bytes(cache, num_seqs, num_q_heads, max_seq_len):
    return int(lib().kvq_decode_workspace_bytes(ctypes.byref(cache.desc), num_seqs, num_q_heads,
                                                max_seq_len))


def paged_decode_attn(cache, q, seq_lens, max_seq_len, block_table, k_codes, k_params, v_codes,
                      v_params, out=None, workspace=None, sm_scale=None, err=None, stream=None):
    """q: float16 CUDA [S][Hq][d]; returns float32 [S][Hq][d]. The workspace
    (``decode_workspace_bytes``) needs no initialisation; without one, one is
    allocated for the call."""
    S, Hq, d = q.shape
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((S, Hq, d), dtype=torch.float32, device=q.device)
    need = decode_workspace_bytes(cache, S, Hq, max_seq_len)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    st = lib().kvq_paged_decode_attn(ctypes.byref(cache.desc), S, Hq, _ptr(q), _ptr(seq_lens),
                                     int(max_seq_len), _ptr(block_table),
                                     int(block_table.shape[1]), float(sm_scale), _ptr(k_codes),
                                     _ptr(k_params), _ptr(v_codes), _ptr(v_params), _ptr(out),
                                     _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _ptr(err), _stream(stream))
    _check("kvq_paged_decode_attn", st)
    return out


def decode_step(cache, q, k_new, v_new, seq_lens, max_seq_len, block_table, k_codes, k_params,
                v_codes, v_params, out=None, workspace=None, sm_scale=None, err=None,
                stream=None):
    """One fused decode step: writes the new token of every sequence (k_new,
    v_new float16 CUDA [S][H][d], or row-strided views with the same row
    layout) at position seq_lens[s] - 1 and returns the attention output
    float32 [S][Hq][d] over seq_lens[s] tokens (lengths include the new
    token). Workspace as for ``paged_decode_attn``."""
    S, Hq, d = q.shape
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((S, Hq, d), dtype=torch.float32, device=q.device)
    need = decode_workspace_bytes(cache, S, Hq, max_seq_len)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    new_stride = k_new.stride(0)
    if v_new.stride(0) != new_stride:
        raise ValueError("k_new and v_new must share the row stride")
    st = lib().kvq_decode_step(ctypes.byref(cache.desc), S, Hq, _ptr(q), _ptr(k_new), _ptr(v_new),
                               int(new_stride), _ptr(seq_lens), int(max_seq_len),
                               _ptr(block_table), int(block_table.shape[1]), float(sm_scale),
                               _ptr(k_codes), _ptr(k_params), _ptr(v_codes), _ptr(v_params),
                               _ptr(out), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _ptr(err),
                               _stream(stream))
    _check("kvq_decode_step", st)
    return out


def decode_fp16_workspace_bytes(cache, num_seqs, num_q_heads, max_seq_len):
    return int(lib().kvq_decode_fp16_workspace_bytes(ctypes.byref(cache.desc), num_seqs,
                                                     num_q_heads, max_seq_len))


def paged_decode_attn_fp16(cache, q, seq_lens, max_seq_len, block_table, k_pages, v_pages,
                           out=None, workspace=None, sm_scale=None, err=None, stream=None):
    """Full-precision baseline over a binary16 paged cache ``k_pages``,
    ``v_pages`` (float16 CUDA [NP][H][P][d], unrotated); q float16 [S][Hq][d];
    returns float32 [S][Hq][d]. Workspace as for ``paged_decode_attn``."""
    S, Hq, d = q.shape
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((S, Hq, d), dtype=torch.float32, device=q.device)
    need = decode_fp16_workspace_bytes(cache, S, Hq, max_seq_len)
    if workspace is None:
        workspace = torch.zeros(max(need, 16), dtype=torch.uint8, device=q.device)
    st = lib().kvq_paged_decode_attn_fp16(ctypes.byref(cache.desc), S, Hq, _ptr(q),
                                          _ptr(seq_lens), int(max_seq_len), _ptr(block_table),
                                          int(block_table.shape[1]), float(sm_scale),
                                          _ptr(k_pages), _ptr(v_pages), _ptr(out),
                                          _ptr(workspace),
                                          workspace.numel() * workspace.element_size(),
                                          _ptr(err), _stream(stream))
    _check("kvq_paged_decode_attn_fp16", st)
    return out


def paged_decode_attn_noalloc(cache, q, seq_lens, max_seq_len, block_table, k_codes, k_params,
                              v_codes, v_params, out=None, sm_scale=None, err=None, stream=None):
    """Decode attention whose scratch is the library's fixed device array
    (for callers that cannot allocate); q: float16 CUDA [S][Hq][d]."""
    S, Hq, d = q.shape
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((S, Hq, d), dtype=torch.float32, device=q.device)
    st = lib().kvq_paged_decode_attn_noalloc(ctypes.byref(cache.desc), S, Hq, _ptr(q),
                                             _ptr(seq_lens), int(max_seq_len), _ptr(block_table),
                                             int(block_table.shape[1]), float(sm_scale),
                                             _ptr(k_codes), _ptr(k_params), _ptr(v_codes),
                                             _ptr(v_params), _ptr(out), _ptr(err),
                                             _stream(stream))
    _check("kvq_paged_decode_attn_noalloc", st)
    return out


def dequantize_pages(cache, seq_lens, max_seq_len, block_table, codes, params, unrotate=False,
                     out_fp32=True, out=None, err=None, stream=None):
    S = int(block_table.shape[0])
    if out is None:
        out = torch.zeros((S, max_seq_len, cache.H, cache.d),
                          dtype=torch.float32 if out_fp32 else torch.float16,
                          device=codes.device)
    st = lib().kvq_dequantize_pages(ctypes.byref(cache.desc), S, _ptr(seq_lens), int(max_seq_len),
                                    _ptr(block_table), int(block_table.shape[1]), _ptr(codes),
                                    _ptr(params), int(bool(unrotate)), int(bool(out_fp32)),
                                    _ptr(out), _ptr(err), _stream(stream))
    _check("kvq_dequantize_pages", st)
    return out


def version():
    return lib().kvq_version().decode()
