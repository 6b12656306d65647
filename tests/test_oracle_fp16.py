"""Pins the oracle's binary16 conversions to library routines and to the
IEEE-754 ordering relations.

RN is compared with numpy's and torch's float32 -> float16 casts (both
round-to-nearest-even), over a strided sweep of all 2^32 binary32 bit
patterns plus every binary16 rounding boundary and its binary32 neighbours.
RD and RU are pinned by RD(x) <= x <= RU(x), equality with RN when x is a
binary16 value, and adjacency otherwise.
"""

import numpy as np
import pytest
import torch

import oracle


def _boundary_floats():
    """Every finite binary16 value, every midpoint between neighbours, and the
    binary32 values one ulp either side of each, as float32."""
    h = np.arange(0, 0x7C00, dtype=np.uint16)              # +0 .. max finite
    v = h.view(np.float16).astype(np.float64)
    mids = (v[:-1] + v[1:]) / 2                             # exact in binary32
    mids = np.concatenate([mids, [65520.0]])                # overflow boundary
    base = np.concatenate([v, mids]).astype(np.float32)
    up = np.nextafter(base, np.float32(np.inf))
    dn = np.nextafter(base, np.float32(-np.inf))
    allp = np.concatenate([base, up, dn])
    return np.concatenate([allp, -allp]).astype(np.float32)


def _strided_patterns(stride=4099):
    bits = np.arange(0, 1 << 32, stride, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    return x[~np.isnan(x)]


def test_half_to_double_all_patterns():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.half_bits_to_double(h)
    ref = h.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signs of zeros
    assert np.signbit(got[0x8000]) and not np.signbit(got[0])


@pytest.mark.parametrize("source", ["boundaries", "strided"])
def test_half_rn_matches_library_casts(source):
    x = _boundary_floats() if source == "boundaries" else _strided_patterns()
    got = oracle.float_to_half_bits(x, oracle.RN)
    with np.errstate(over="ignore"):
        ref_np = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref_np)
    ref_t = torch.from_numpy(x).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref_t)


def _next_up_f16(bits):
    """Next binary16 toward +inf (as bits), for finite non-NaN inputs."""
    v = bits.view(np.float16)
    with np.errstate(over="ignore"):
        return np.nextafter(v, np.float16(np.inf)).view(np.uint16)


@pytest.mark.parametrize("source", ["boundaries", "strided"])
def test_half_directed_rounding_brackets(source):
    x = _boundary_floats() if source == "boundaries" else _strided_patterns()
    x = x[np.isfinite(x)]
    rd = oracle.float_to_half_bits(x, oracle.RD)
    ru = oracle.float_to_half_bits(x, oracle.RU)
    rn = oracle.float_to_half_bits(x, oracle.RN)
    xd = x.astype(np.float64)
    vd = rd.view(np.float16).astype(np.float64)
    vu = ru.view(np.float16).astype(np.float64)
    # RD(x) <= x <= RU(x), with infinities only where x is beyond the range
    assert np.all(vd <= xd) and np.all(vu >= xd)
    exact = vd == xd
    # exactly representable -> all three modes agree (sign of zero included)
    assert np.array_equal(rd[exact], rn[exact])
    assert np.array_equal(ru[exact & (vu == xd)], rn[exact & (vu == xd)])
    assert np.all(vu[exact] == xd[exact])
    # otherwise RD and RU are adjacent binary16 values
    ne = ~exact
    assert np.array_equal(_next_up_f16(rd[ne]).view(np.float16).astype(np.float64), vu[ne])
    # RN is one of the two
    vn = rn.view(np.float16).astype(np.float64)
    assert np.all((vn == vd) | (vn == vu) | (np.abs(xd) >= 65520))


def test_half_directed_rounding_hand_cases():
    f = lambda x, m: int(oracle.float_to_half_bits(np.array([x], np.float32), m)[0])
    # 0.2 lies between 1638 * 2^-13 and 1639 * 2^-13
    assert f(0.2, oracle.RD) == 0x3266 and f(0.2, oracle.RU) == 0x3267
    assert f(-0.2, oracle.RD) == 0xB267 and f(-0.2, oracle.RU) == 0xB266
    # beyond the largest finite value
    assert f(70000.0, oracle.RD) == 0x7BFF and f(70000.0, oracle.RU) == 0x7C00
    assert f(-70000.0, oracle.RU) == 0xFBFF and f(-70000.0, oracle.RD) == 0xFC00
    # tiny positive values round up to the smallest subnormal / down to +0
    assert f(1e-30, oracle.RU) == 0x0001 and f(1e-30, oracle.RD) == 0x0000
    assert f(-1e-30, oracle.RD) == 0x8001 and f(-1e-30, oracle.RU) == 0x8000
