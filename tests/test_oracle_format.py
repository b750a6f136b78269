"""Pins of the oracle's number formats against things other than itself:
the pages' E2M1 definition (hand-worked golden tables), the ml_dtypes and torch
implementations of float4_e2m1fn / float8_e4m3fn / bfloat16 rounding, and exact
rational rounding.

Format source: "LongLive-2.0：用 NVFP4 并行底座做长视频生成" (yingwang.github.io
reading note), section 二 方法 / "NVFP4 量化格式".
"""
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle


def test_e2m1_decode_golden(golden):
    rows = golden("e2m1_grid.txt")
    assert len(rows) == 16
    for code, val in rows:
        v = oracle.e2m1_value(int(code))
        assert v == float(val)
        assert np.signbit(v) == val.startswith("-")


def test_e2m1_decode_matches_ml_dtypes():
    lib_vals = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    for c in range(16):
        v = oracle.e2m1_value(c)
        assert v == lib_vals[c] and np.signbit(v) == np.signbit(lib_vals[c])


def test_e2m1_encode_golden_ties(golden):
    for x, code in golden("e2m1_rne.txt"):
        assert oracle.e2m1_encode(float(np.float32(x))) == int(code), x


def _e2m1_probe_points():
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    pts = []
    for lo, hi in zip(grid[:-1], grid[1:]):
        mid = np.float32((lo + hi) / 2)
        for v in (lo, hi, mid):
            v = np.float32(v)
            pts += [v, np.nextafter(v, np.float32(0)), np.nextafter(v, np.float32(10))]
    pts += [np.float32(6.0), np.float32(6.5), np.float32(7.0), np.float32(1e30), np.float32(1e-40)]
    g = np.random.default_rng(5)
    pts += list(g.uniform(-7, 7, 4000).astype(np.float32))
    pts = np.array(pts, np.float32)
    return np.concatenate([pts, -pts])


def test_e2m1_encode_matches_ml_dtypes():
    pts = _e2m1_probe_points()
    ref = pts.astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    got = np.array([oracle.e2m1_encode(float(p)) for p in pts], np.uint8)
    bad = np.nonzero(ref != got)[0]
    assert bad.size == 0, [(pts[i], ref[i], got[i]) for i in bad[:10]]


def test_e4m3_decode_matches_torch_and_ml_dtypes():
    codes = torch.arange(256, dtype=torch.uint8)
    tv = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mv = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for c in range(256):
        v = oracle.e4m3_value(c)
        if np.isnan(tv[c]):
            assert np.isnan(v) and np.isnan(mv[c])
        else:
            assert v == tv[c] == mv[c]
    # the largest finite E4M3 value is 448 (code 0x7E); 0x7F is NaN
    assert oracle.e4m3_value(0x7E) == 448.0 and np.isnan(oracle.e4m3_value(0x7F))


def test_e4m3_encode_matches_libraries_in_range():
    vals = [np.float32(oracle.e4m3_value(c)) for c in range(127)]
    pts = []
    for lo, hi in zip(vals[:-1], vals[1:]):
        mid = np.float32((float(lo) + float(hi)) / 2)
        for v in (lo, mid):
            pts += [v, np.nextafter(v, np.float32(0)), np.nextafter(v, np.float32(1e9))]
    pts += [np.float32(2.0 ** -10), np.float32(2.0 ** -11), np.float32(1e-30), np.float32(0.0),
            np.float32(448.0), np.float32(460.0), np.float32(463.99)]
    g = np.random.default_rng(7)
    pts += list(np.exp(g.uniform(np.log(1e-4), np.log(460.0), 5000)).astype(np.float32))
    pts = np.array(pts, np.float32)
    ref_m = pts.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    ref_t = torch.from_numpy(pts).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(p)) for p in pts], np.uint8)
    assert (ref_m == ref_t).all()
    bad = np.nonzero(ref_m != got)[0]
    assert bad.size == 0, [(pts[i], ref_m[i], got[i]) for i in bad[:10]]


@pytest.mark.parametrize("r", [448.0, 449.0, 464.0, 465.0, 1000.0, 3.0e38])
def test_e4m3_encode_saturates(r):
    # R3: the libraries turn values past 464 into NaN; the block scale saturates at 448.
    assert oracle.e4m3_encode(r) == 0x7E


def test_bf16_from_f32_matches_torch():
    g = np.random.default_rng(3)
    x = np.concatenate([g.standard_normal(20000).astype(np.float32) * np.float32(1e3),
                        g.standard_normal(2000).astype(np.float32) * np.float32(1e-39),
                        np.array([0.0, -0.0, 1.0, 65504.0, 3.0e38], np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f64_to_bf16(float(v)) for v in x], np.uint16)
    assert (ref == got).all()


def _bf16_exact(x: Fraction) -> float:
    """Nearest-even bf16 of an exact rational, by brute force over neighbours."""
    if x == 0:
        return 0.0
    sgn = -1 if x < 0 else 1
    a = abs(x)
    e = 0
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q = max(e - 7, -133)
    step = Fraction(2) ** q
    k = a / step
    lo = k.numerator // k.denominator
    rem = k - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return sgn * float(lo * step)


def test_bf16_from_f64_single_rounding():
    # binary64 -> bf16 must round once (no detour through binary32).
    g = np.random.default_rng(11)
    xs = list(g.standard_normal(3000) * 10.0)
    # values just above a bf16 midpoint by less than a binary32 ulp: a double
    # rounding through binary32 would land on the tie and round to even.
    for m in range(128, 256, 7):
        mid = (m + 0.5) * 2.0 ** -7
        xs += [mid + 2.0 ** -40, mid - 2.0 ** -40, mid]
    for x in xs:
        want = _bf16_exact(Fraction(x))
        got = oracle.bf16_to_f32(oracle.f64_to_bf16(x))
        assert got == want, (x, got, want)
