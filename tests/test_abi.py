"""The C-ABI library builds, loads without a GPU, exports every function that
include/kvq.h declares, and rejects bad arguments on the host (these calls
return before any CUDA call, so no GPU is needed)."""

import ctypes
import os
import re

import pytest

from bit_rotated_kv_block_b200 import build, kvq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return kvq.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(kvq_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_every_declared_function_is_exported(L):
    names = declared_functions()
    assert "kvq_quantize_append" in names and "kvq_paged_decode_attn" in names
    assert "kvq_dequantize_pages" in names and "kvq_decode_workspace_bytes" in names
    for n in names:
        assert hasattr(L, n), n
        assert n in kvq.SIGNATURES, n


def test_status_strings_and_version(L):
    assert kvq.version().startswith("libkvq")
    for code, name in kvq.STATUS.items():
        assert L.kvq_status_string(code).decode() == name


def _desc(**kw):
    base = dict(head_dim=128, num_kv_heads=8, page_size=16, num_pages=16, rot_kind=1,
                rot_block=128, quat=None)
    base.update(kw)
    return kvq.CacheDesc(**base)


def _append(L, desc, T=1, k=16, v=16, stride=1024, seq=16, pos=16, S=1, bt=16, bts=1, pools=16):
    P = ctypes.c_void_p
    return L.kvq_quantize_append(ctypes.byref(desc), T, P(k) if k else None, P(v) if v else None,
                                 stride, P(seq) if seq else None, P(pos) if pos else None, S,
                                 P(bt) if bt else None, bts, P(pools), P(pools), P(pools),
                                 P(pools), None, None)


def test_host_validation_codes(L):
    OK, INV, UNS, MIS = 0, 1, 2, 3
    assert _append(L, _desc(), T=0) == OK                       # empty batch: no launch
    assert _append(L, _desc(head_dim=100)) == UNS
    assert _append(L, _desc(page_size=24)) == UNS
    assert _append(L, _desc(rot_block=96)) == INV               # not a power of two
    assert _append(L, _desc(rot_block=8)) == UNS                # below the supported blocks
    assert _append(L, _desc(rot_block=256)) == INV              # wider than head_dim
    assert _append(L, _desc(rot_kind=2)) == INV                 # quaternion without a table
    assert _append(L, _desc(rot_kind=7)) == INV
    assert _append(L, _desc(num_kv_heads=0)) == INV
    assert _append(L, _desc(), k=0) == INV                      # null input
    assert _append(L, _desc(), stride=1000) == INV              # stride < H * d
    assert _append(L, _desc(), stride=1028) == MIS              # stride not a multiple of 8
    assert _append(L, _desc(), k=24) == MIS                     # misaligned pointer
    assert _append(L, _desc(), T=-1) == INV
    desc = _desc()
    assert L.kvq_decode_workspace_bytes(ctypes.byref(desc), 0, 32, 100) == 0
    assert L.kvq_decode_workspace_bytes(ctypes.byref(desc), 2, 30, 100) == 0   # Hq % H != 0


def test_host_validation_of_step_and_baseline(L):
    """kvq_decode_step and kvq_paged_decode_attn_fp16 reject bad arguments on
    the host before touching any device memory (fake pointers, no launch)."""
    OK, INV, UNS, MIS = 0, 1, 2, 3
    desc = _desc()
    P = ctypes.c_void_p
    good = 1 << 20  # a 16-byte aligned fake address

    def step(q=good, k=good, v=good, stride=4096, lens=good, Hq=32, ws=good):
        return L.kvq_decode_step(ctypes.byref(desc), 2, Hq, P(q), P(k), P(v), stride, P(lens), 100,
                                 P(good), 8, 0.1, P(good), P(good), P(good), P(good), P(good),
                                 P(ws), 0, None, None)

    assert step(Hq=30) == INV            # query heads not a multiple of KV heads
    assert step(Hq=8 * 16) == UNS        # GQA group above 8
    assert step(k=0) == INV              # null new-token rows
    assert step(stride=100) == INV       # row stride below H * d
    assert step(stride=1028 + 4096) == MIS  # stride not a multiple of 8
    assert step(v=good + 8) == MIS       # misaligned rows
    assert step(q=good + 4) == MIS
    d16 = _desc()
    assert L.kvq_paged_decode_attn_fp16(ctypes.byref(d16), 2, 30, P(good), P(good), 100, P(good),
                                        8, 0.1, P(good), P(good), P(good), P(good), 0, None,
                                        None) == INV
    assert L.kvq_paged_decode_attn_fp16(ctypes.byref(d16), 2, 32, P(good), P(good), 100, P(good),
                                        8, 0.1, P(good + 8), P(good), P(good), P(good), 0, None,
                                        None) == MIS
    assert L.kvq_decode_fp16_workspace_bytes(ctypes.byref(d16), 0, 32, 100) == 0



def _prototypes():
    """name -> (return type, [parameter types]) parsed from include/kvq.h."""
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for m in re.finditer(r"^\s*((?:const\s+)?[A-Za-z_]\w*\s*\**)\s*\b(kvq_\w+)\s*\(([^)]*)\)\s*;",
                         text, flags=re.M):
        ret, name, params = m.group(1).strip(), m.group(2), m.group(3).strip()
        types = []
        if params and params != "void":
            for p in params.split(","):
                p = " ".join(p.split())
                ptr = p.count("*")
                base = re.sub(r"\b(const)\b", "", p).replace("*", " ").split()
                # drop the parameter name (the last identifier) when present
                if len(base) > 1:
                    base = base[:-1]
                types.append((" ".join(base), ptr))
        out[name] = (ret, types)
    return out


_CTYPE = {("int32_t", 0): ctypes.c_int32, ("int64_t", 0): ctypes.c_int64,
          ("float", 0): ctypes.c_float, ("size_t", 0): ctypes.c_size_t, ("int", 0): ctypes.c_int}


def test_binding_signatures_match_the_header():
    protos = _prototypes()
    assert set(protos) == set(declared_functions())
    for name, (res, args) in kvq.SIGNATURES.items():
        ret, params = protos[name]
        assert len(params) == len(args), (name, len(params), len(args))
        for i, ((base, ptr), a) in enumerate(zip(params, args)):
            if ptr:
                assert a in (ctypes.c_void_p, ctypes.c_char_p), (name, i, base, a)
            else:
                want = _CTYPE[(base, 0)]
                assert ctypes.sizeof(a) == ctypes.sizeof(want), (name, i, base, a)
                assert (a == ctypes.c_float) == (want == ctypes.c_float), (name, i, base, a)
        if "*" in ret:
            assert res in (ctypes.c_char_p, ctypes.c_void_p), name
        else:
            assert ctypes.sizeof(res) == ctypes.sizeof(_CTYPE[(ret.replace("const", "").strip(), 0)]), name


def test_cache_desc_mirrors_the_header_struct():
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    body = re.search(r"typedef struct\s*\{(.*?)\}\s*kvq_cache_desc\s*;", text, flags=re.S).group(1)
    fields = [f.split() for f in body.replace("*", " * ").split(";") if f.strip()]
    names = [f[-1] for f in fields]
    assert names == [n for n, _ in kvq.CacheDesc._fields_]
    for f, (n, t) in zip(fields, kvq.CacheDesc._fields_):
        if "*" in f:
            assert t is ctypes.c_void_p, n
        else:
            assert f[-2] == "int32_t" and t is ctypes.c_int32, n
    # the C layout on a 64-bit host: six int32, two pointers, two int32, a pointer
    assert kvq.CacheDesc.quat.offset == 24 and kvq.CacheDesc.rope.offset == 32
    assert kvq.CacheDesc.rope_max_pos.offset == 40 and kvq.CacheDesc.format.offset == 44
    assert kvq.CacheDesc.levels.offset == 48 and ctypes.sizeof(kvq.CacheDesc) == 56
