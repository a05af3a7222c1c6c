"""Pins for the oracle's element and scale codecs (CPU only).

Each check ties the oracle to something other than itself: the value set the
pages print, the format maxima they print, and brute-force nearest searches
written here independently of the oracle's arithmetic encoders.
"""
import math
import struct

import numpy as np
import pytest

from conftest import golden_dict, read_golden


def f32(x):
    return struct.unpack("<f", struct.pack("<f", x))[0]


def f32_next(x, n=1):
    b = struct.unpack("<I", struct.pack("<f", x))[0]
    return struct.unpack("<f", struct.pack("<I", b + n))[0]


def f32_prev(x, n=1):
    return f32_next(x, -n)


# ------------------------------------------------------------------ E2M1
def test_e2m1_decodes_to_printed_grid(orc):
    grid = sorted(float(r[0]) for r in read_golden("e2m1_grid.txt"))
    vals = sorted(set(orc.e2m1_value(c) for c in range(16)))
    assert vals == grid
    # positive codes 0..7 increasing, code 8+i is the negation of code i
    pos = [orc.e2m1_value(c) for c in range(8)]
    assert pos == sorted(pos)
    for c in range(8):
        assert orc.e2m1_value(c | 8) == -pos[c]
    assert max(abs(v) for v in vals) == golden_dict("format_maxima.txt")["M_FP4"]


def _brute_e2m1(v):
    """Nearest grid magnitude by exhaustive search; equal distances go to the
    code with mantissa bit 0; sign from the sign bit."""
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    a = abs(v)
    dists = [abs(a - m) for m in mags]
    best = min(dists)
    cands = [i for i, d in enumerate(dists) if d == best]
    even = [i for i in cands if i % 2 == 0]
    code = even[0] if even else cands[0]
    return code | (8 if math.copysign(1.0, v) < 0 else 0)


def test_e2m1_encode_matches_brute_force_at_every_tie(orc):
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    pts = []
    for m in mids:
        for k in range(-3, 4):
            pts.append(f32_next(m, k))
    pts += [0.0, 6.0, 6.5, 7.0, 100.0, 1e30, 1e-30, 0.4999, 5.9999]
    for v in pts:
        for s in (1.0, -1.0):
            x = f32(s * v)
            assert orc.e2m1_encode(x) == _brute_e2m1(x), x


def test_e2m1_tie_table(orc):
    # the tie cases spelled out: x.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2,
    # 2.5 -> 2, 3.5 -> 4, 5 -> 4 (value), i.e. toward the even code
    table = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for v, want in table.items():
        assert orc.e2m1_value(orc.e2m1_encode(v)) == want
        assert orc.e2m1_value(orc.e2m1_encode(-v)) == -want


def test_e2m1_random_against_brute(orc):
    rng = np.random.default_rng(7)
    xs = np.concatenate([rng.uniform(-8, 8, 20000), rng.normal(0, 2, 20000)]).astype(np.float32)
    for x in xs:
        assert orc.e2m1_encode(float(x)) == _brute_e2m1(float(x))


def test_e2m1_saturates_and_keeps_sign(orc):
    assert orc.e2m1_encode(1e9) == 7
    assert orc.e2m1_encode(-1e9) == 15
    assert orc.e2m1_encode(float("inf")) == 7
    assert orc.e2m1_encode(-0.1) == 8  # small negatives keep the sign bit
    assert orc.e2m1_encode(-0.0) == 8


# ------------------------------------------------------------------ E4M3
def _e4m3_table():
    """All finite non-negative E4M3 values from the bit-field definition
    (bias 7, 3 mantissa bits, exponent field 0 subnormal), codes 0..0x7E."""
    out = []
    for c in range(0x7F):
        e, m = c >> 3, c & 7
        v = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
        out.append(v)
    return out


def _brute_e4m3(t):
    tab = _e4m3_table()
    if t >= tab[-1]:
        return 0x7E
    dists = [abs(t - v) for v in tab]
    best = min(dists)
    cands = [i for i, d in enumerate(dists) if d == best]
    even = [i for i in cands if i % 2 == 0]
    return even[0] if even else cands[0]


def test_e4m3_range(orc):
    tab = _e4m3_table()
    for c in range(0x7F):
        assert orc.e4m3_decode(c) == tab[c]
    assert orc.e4m3_decode(0x7E) == golden_dict("format_maxima.txt")["M_FP8"] == 448.0
    assert orc.e4m3_decode(1) == 2.0 ** -9
    assert all(tab[i] < tab[i + 1] for i in range(len(tab) - 1))  # monotone


def test_e4m3_encode_midpoints_against_brute(orc):
    tab = _e4m3_table()
    pts = []
    for i in range(len(tab) - 1):
        mid = (tab[i] + tab[i + 1]) / 2  # exact in double, representable in fp32
        for k in range(-2, 3):
            pts.append(f32_next(f32(mid), k))
    pts += [f32(v) for v in tab] + [448.0, 449.0, 464.0, 480.0, 1e6, 0.0, 1e-12]
    for t in pts:
        assert orc.e4m3_encode(t) == _brute_e4m3(t), t


def test_e4m3_encode_random_against_brute(orc):
    rng = np.random.default_rng(11)
    ts = (2.0 ** rng.uniform(-12, 10, 100000)).astype(np.float32)
    tab = np.array(_e4m3_table())
    for t in ts[:20000]:
        assert orc.e4m3_encode(float(t)) == _brute_e4m3(float(t))
    # vectorised brute force for the rest
    t = ts.astype(np.float64)
    d = np.abs(t[:, None] - tab[None, :])
    idx = d.argmin(axis=1)  # lower index on a tie
    nxt = np.minimum(idx + 1, 126)
    rows = np.arange(t.size)
    tie_up = (idx < 126) & (d[rows, nxt] == d[rows, idx])
    codes = np.where(tie_up & (idx % 2 == 1), idx + 1, idx)
    codes[t >= 448] = 0x7E
    got = np.array([orc.e4m3_encode(float(x)) for x in ts])
    assert np.array_equal(got, codes)


# ------------------------------------------------------------------ bf16
def test_bf16_rne_ties_by_hand(orc):
    # 1 + 2^-8 is the midpoint of 1 and 1 + 2^-7: ties to the even mantissa (1.0)
    assert orc.bf16_rne(1.0 + 2.0 ** -8) == 0x3F80
    # 1 + 3*2^-8 is the midpoint of 1+2^-7 (odd) and 1+2^-6 (even)
    assert orc.bf16_rne(1.0 + 3 * 2.0 ** -8) == 0x3F82
    assert orc.bf16_rne(f32_next(1.0 + 2.0 ** -8)) == 0x3F81
    assert orc.bf16_rne(-2.0) == 0xC000


def test_bf16_rne_matches_torch(orc):
    import torch
    rng = np.random.default_rng(3)
    xs = rng.normal(0, 10, 5000).astype(np.float32)
    want = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([orc.bf16_rne(float(x)) for x in xs], dtype=np.uint16)
    assert np.array_equal(got, want)


# ------------------------------------------------------------------ range casts
def test_range_casts_equal_the_scalar_casts(orc):
    """encode_bits (the oracle's side of the GPU conversion sweeps) is the
    scalar casts applied to consecutive bit patterns: checked on ranges that
    hold every E2M1 tie, the E4M3 saturation point and signed zeros."""
    for target, first, n in ((0, 0x3E000000, 4096), (0, 0x40A00000 - 2048, 4096),
                             (0, 0x7FFFF000, 8192), (1, 0x43DFF000, 8192),
                             (1, 0x3A000000 - 100, 200), (1, 0x7F7FFFF0, 17)):
        got = orc.encode_bits(target, first, n)
        bits = (np.arange(n, dtype=np.uint64) + first).astype(np.uint32)
        vals = bits.view(np.float32)
        f = orc.e2m1_encode if target == 0 else orc.e4m3_encode
        want = np.array([f(float(v)) if np.isfinite(v) else f(float(v)) for v in vals], np.uint8)
        assert np.array_equal(got, want), (target, hex(first))
