"""Pins for the oracle's quantizers (CPU only): the 6-rule, the 4-vs-6 pick,
global scale, round trips, zero / constant blocks, 2D tiles, the transposing
variant, scale-factor layouts and the KV storage accounting."""
import numpy as np
import pytest

from conftest import golden_dict

GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def e4m3_values():
    out = []
    for c in range(0x7F):
        e, m = c >> 3, c & 7
        out.append(m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    return out


def unpack(codes, n):
    c = np.asarray(codes, dtype=np.uint8).reshape(-1)
    out = np.empty(c.size * 2, dtype=np.uint8)
    out[0::2] = c & 15
    out[1::2] = c >> 4
    return out[:n]


def decode_codes(q):
    mag = np.array(GRID)[q & 7]
    return np.where(q & 8, -mag, mag)


# ------------------------------------------------------------- global scale
def test_global_scale_maps_tensor_max_to_fp8_max(orc):
    M = golden_dict("format_maxima.txt")
    rng = np.random.default_rng(0)
    for trial in range(20):
        x = (rng.standard_normal((8, 64)) * 10 ** rng.uniform(-3, 3)).astype(np.float32)
        codes, sf, alpha = orc.quantize_1d(x, four_over_six=False)
        amax = float(np.abs(x).max())
        assert alpha == np.float32(np.float32(amax) / np.float32(M["M_FP4"] * M["M_FP8"]))
        # the block holding the max gets the largest E4M3 scale, code 0x7E (=448)
        r, c = np.unravel_index(np.abs(x).argmax(), x.shape)
        assert sf[r * (x.shape[1] // 16) + c // 16] == 0x7E
        # and its max element is encoded as +-6 (the 6-rule)
        q = unpack(codes[r], x.shape[1])[c]
        assert abs(decode_codes(np.array([q]))[0]) == M["M_FP4"]


def test_global_scale_all_zero(orc):
    x = np.zeros((4, 32), np.float32)
    codes, sf, alpha = orc.quantize_1d(x)
    assert alpha == 1.0
    assert not codes.any() and not sf.any()


# ------------------------------------------------------------- the 6-rule
def test_six_rule_closed_form(orc):
    """bmax = alpha * 6 * d for a representable d gives scale d and code +-6."""
    alpha = 0.125  # power of two: every product below is exact
    rng = np.random.default_rng(1)
    for code in [8, 20, 37, 56, 70, 100, 119]:
        d = orc.e4m3_decode(code)
        bmax = alpha * 6 * d
        y = rng.uniform(-0.9, 0.9, 16) * bmax
        y[5] = -bmax
        codes, sf, a = orc.quantize_1d(y[None, :].astype(np.float32), four_over_six=False,
                                       alpha_in=alpha)
        assert sf[0] == code
        assert unpack(codes, 16)[5] == 15  # -6


# ------------------------------------------------------------- 4-vs-6 pick
def _encode_with_scale(y, s):
    """Encode block y with scale s: nearest grid value of y/s (fp64 here)."""
    a = np.abs(y) / s
    mags = np.array(GRID)
    idx = np.abs(a[:, None] - mags[None, :]).argmin(axis=1)
    return np.sign(y) * mags[idx] * s


def test_four_over_six_pick_is_better_candidate_brute_force(orc):
    """On tiny blocks, enumerate every positive E4M3 scale (brute force): the
    oracle's chosen scale must be one of the two candidates of the scale
    search and its (fp64) error must not exceed the other candidate's beyond
    fp32 rounding."""
    rng = np.random.default_rng(2)
    alpha = 1.0
    scales = [v for v in e4m3_values() if v > 0]
    better_elsewhere = 0
    n = 400
    for _ in range(n):
        y = (rng.standard_normal(16) * rng.uniform(0.5, 40)).astype(np.float32)
        if rng.random() < 0.3:
            y[rng.integers(16)] *= 6
        codes, sf, _ = orc.quantize_1d(y[None, :], four_over_six=True, alpha_in=alpha)
        bmax = float(np.abs(y).max())
        d6 = orc.e4m3_decode(orc.e4m3_encode(np.float32(bmax / 6)))
        d4 = orc.e4m3_decode(orc.e4m3_encode(np.float32(bmax / 4)))
        d_pick = orc.e4m3_decode(int(sf[0]))
        assert d_pick in (d6, d4)
        yd = y.astype(np.float64)
        err = {d: float(((yd - _encode_with_scale(yd, d)) ** 2).sum()) for d in (d6, d4)}
        other = d4 if d_pick == d6 else d6
        assert err[d_pick] <= err[other] * (1 + 1e-5) + 1e-30
        # decoded block equals the nearest-grid encoding under the chosen scale,
        # except possibly where y/s sits within fp32 rounding of a midpoint
        q = unpack(codes, 16)
        got = decode_codes(q) * d_pick
        want = _encode_with_scale(yd, d_pick)
        ratio = np.abs(yd) / d_pick
        mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
        near = (np.abs(ratio[:, None] - mids[None, :]) <= mids * 2 ** -22).any(axis=1)
        assert np.all((got == want) | near)
        full = min(float(((yd - _encode_with_scale(yd, s)) ** 2).sum()) for s in scales)
        if full < min(err.values()) * (1 - 1e-6):
            better_elsewhere += 1
    # informational: the two-candidate search is not the global optimum
    print("blocks where another E4M3 scale beats both candidates:", better_elsewhere, "/", n)


def test_four_over_six_prefers_four_near_three_quarters(orc):
    """Values near 75% of the block max: the max->4 encoding puts FP4 value 3
    at 75% of the max, the 6-rule cannot (printed fractions in the fixture)."""
    g = golden_dict("four_over_six.txt")
    assert abs(3.0 / 4.0 - g["four_rule_value3_fraction"]) < 1e-12
    assert abs(3.0 / 6.0 - g["six_rule_value3_fraction"]) < 1e-12
    assert abs(4.0 / 6.0 - g["six_rule_next_below_fraction"]) < 1e-3
    y = np.full(16, 0.75, np.float32) * 8.0
    y[0] = 8.0
    y[1::2] *= -1
    c6, s6, _ = orc.quantize_1d(y[None, :], four_over_six=False, alpha_in=1.0)
    c46, s46, _ = orc.quantize_1d(y[None, :], four_over_six=True, alpha_in=1.0)
    assert orc.e4m3_decode(int(s46[0])) == 2.0  # 8 / 4
    assert orc.e4m3_decode(int(s6[0])) != 2.0
    deq = decode_codes(unpack(c46, 16)) * 2.0
    assert np.array_equal(deq, y.astype(np.float64))  # exact under max->4


def test_four_over_six_prefers_six_for_outlier_block(orc):
    y = np.array([12.0] + [0.3, -0.2, 0.1, 1.9, -2.1, 0.05, 3.1, -0.7, 0.0, 0.4, 1.0,
                           -1.2, 0.8, 0.6, -0.45], np.float32)
    _, s, _ = orc.quantize_1d(y[None, :], four_over_six=True, alpha_in=1.0)
    assert orc.e4m3_decode(int(s[0])) == 2.0  # 12 / 6


def test_four_over_six_off_is_six_rule(orc):
    rng = np.random.default_rng(4)
    x = rng.standard_normal((16, 64)).astype(np.float32)
    _, s, a = orc.quantize_1d(x, four_over_six=False)
    blocks = np.abs(x).reshape(16, 4, 16).max(axis=2).reshape(-1)
    for b, code in zip(blocks, s):
        t = np.float32(np.float32(np.float32(b) / np.float32(a)) / np.float32(6))
        assert code == orc.e4m3_encode(float(t))


# ------------------------------------------------------------- round trips
def test_round_trip_idempotent(orc):
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((32, 128)) * 3).astype(np.float32)
    x[:, 7] *= 30
    c1, s1, a = orc.quantize_1d(x)
    d1, _ = orc.dequantize(c1, s1, a, 32, 128)
    c2, s2, _ = orc.quantize_1d(d1, alpha_in=a)
    d2, _ = orc.dequantize(c2, s2, a, 32, 128)
    assert np.array_equal(d1, d2)
    changed = int((c1 != c2).sum())
    print("code bytes changed by requantization (4/6 ties):", changed)


def test_zero_and_constant_blocks(orc):
    x = np.zeros((3, 48), np.float32)
    x[1, 16:32] = 2.5
    x[2, 32:48] = -0.3
    x[2, 0:16] = 9.0
    c, s, a = orc.quantize_1d(x)
    assert s[0] == 0 and s[1] == 0 and s[2] == 0 and s[5] == 0  # zero blocks
    q = unpack(c.reshape(-1), 3 * 48).reshape(3, 48)
    assert not q[0].any()
    for r, sl in [(1, slice(16, 32)), (2, slice(32, 48)), (2, slice(0, 16))]:
        vals = set(q[r, sl].tolist())
        assert len(vals) == 1 and (list(vals)[0] & 7) in (6, 7)  # all +-4 or all +-6
    d, _ = orc.dequantize(c, s, a, 3, 48)
    assert not d[0].any()
    assert len(set(d[1, 16:32].tolist())) == 1
    assert len(set(d[2, 32:48].tolist())) == 1


# ------------------------------------------------------------- 2D tiles
def test_2d_tile_shares_one_scale(orc):
    rng = np.random.default_rng(6)
    w = (rng.standard_normal((32, 64)) * 0.02).astype(np.float32)
    for layout in (orc.SF_ROWMAJOR, orc.SF_TCGEN05):
        c, s, a = orc.quantize_2d(w, sf_layout=layout)
        for tr in range(2):
            for kb in range(4):
                vals = {int(s[orc.sf_offset(tr * 16 + r, kb, 4, layout)]) for r in range(16)}
                assert len(vals) == 1


def test_2d_equals_1d_with_tile_scale_on_uniform_rows(orc):
    """If all 16 rows of a tile are identical, the tile's max equals each
    row's max, and 16x the same row error keeps the pick: 2D == 1D."""
    rng = np.random.default_rng(8)
    row = rng.standard_normal((1, 64)).astype(np.float32)
    w = np.repeat(row, 16, axis=0)
    c2, s2, a2 = orc.quantize_2d(w)
    c1, s1, a1 = orc.quantize_1d(w)
    assert a1 == a2
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)


def test_2d_pick_brute_force(orc):
    """2D pick against a direct fp64 evaluation of the two tile candidates."""
    rng = np.random.default_rng(9)
    for _ in range(50):
        w = (rng.standard_normal((16, 16)) * rng.uniform(0.01, 5)).astype(np.float32)
        c, s, a = orc.quantize_2d(w, alpha_in=1.0)
        tmax = float(np.abs(w).max())
        d6 = orc.e4m3_decode(orc.e4m3_encode(np.float32(tmax / 6)))
        d4 = orc.e4m3_decode(orc.e4m3_encode(np.float32(tmax / 4)))
        d = orc.e4m3_decode(int(s[0]))
        assert d in (d6, d4)
        wd = w.astype(np.float64).reshape(-1)
        e6 = float(((wd - _encode_with_scale(wd, d6)) ** 2).sum())
        e4 = float(((wd - _encode_with_scale(wd, d4)) ** 2).sum())
        assert (e6 if d == d6 else e4) <= min(e6, e4) * (1 + 1e-5) + 1e-30


# ------------------------------------------------------------- layouts
def test_tcgen05_sf_layout_is_a_bijection_and_matches_rowmajor(orc):
    rows, kb = 200, 12
    n = orc.sf_bytes(rows, kb, orc.SF_TCGEN05)
    assert n == 256 * 12
    offs = [orc.sf_offset(r, k, kb, orc.SF_TCGEN05) for r in range(256) for k in range(kb)]
    assert sorted(offs) == list(range(n))
    # a 128x4 atom: row r at (r%32)*16 + (r//32)*4 within 512 bytes
    assert orc.sf_offset(0, 0, kb, 1) == 0
    assert orc.sf_offset(1, 0, kb, 1) == 16
    assert orc.sf_offset(32, 0, kb, 1) == 4
    assert orc.sf_offset(0, 1, kb, 1) == 1
    assert orc.sf_offset(0, 4, kb, 1) == 512
    assert orc.sf_offset(128, 0, kb, 1) == 512 * 3
    rng = np.random.default_rng(10)
    x = rng.standard_normal((rows, kb * 16)).astype(np.float32)
    c0, s0, a0 = orc.quantize_1d(x, sf_layout=orc.SF_ROWMAJOR)
    c1, s1, a1 = orc.quantize_1d(x, sf_layout=orc.SF_TCGEN05)
    assert np.array_equal(c0, c1)
    for r in range(rows):
        for k in range(kb):
            assert s0[r * kb + k] == s1[orc.sf_offset(r, k, kb, 1)]
    # padding rows are zero
    pad = [orc.sf_offset(r, k, kb, 1) for r in range(rows, 256) for k in range(kb)]
    assert not s1[pad].any()


# ------------------------------------------------------------- transposing
def test_transposed_quantize_equals_quantize_of_transpose(orc):
    rng = np.random.default_rng(12)
    x = rng.standard_normal((64, 48)).astype(np.float32)
    for rht in (False, True):
        ct, st, at = orc.quantize_1d(x, rht=rht, mask=0x5A3C, block_axis=1)
        cr, sr, ar = orc.quantize_1d(np.ascontiguousarray(x.T), rht=rht, mask=0x5A3C)
        assert at == ar and np.array_equal(ct, cr) and np.array_equal(st, sr)


# ------------------------------------------------------------- KV accounting
def test_kv_storage_ratio(orc):
    g = golden_dict("kv_compression.txt")
    rows, d = 24 * 40, 128
    rng = np.random.default_rng(13)
    x = rng.standard_normal((rows, d)).astype(np.float32)
    c, s, _ = orc.quantize_1d(x)
    per_elem = (c.nbytes + s.nbytes) / (rows * d)
    assert per_elem == g["bytes_per_element_nvfp4"]
    ratio = g["bytes_per_element_bf16"] / per_elem
    assert abs(ratio - g["ratio_printed"]) < g["ratio_tolerance"]


def test_dequant_bf16_is_rounded_fp32(orc):
    rng = np.random.default_rng(14)
    x = rng.standard_normal((8, 64)).astype(np.float32)
    c, s, a = orc.quantize_1d(x)
    d32, d16 = orc.dequantize(c, s, a, 8, 64)
    import torch
    want = torch.from_numpy(d32).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    assert np.array_equal(d16, want)
    # the reconstruction identity X^ = X^_FP4 * a_FP8 * a_FP32, term by term in fp64
    q = unpack(c.reshape(-1), 8 * 64).reshape(8, 64)
    dsc = np.array([orc.e4m3_decode(int(v)) for v in s]).reshape(8, 4)
    ref = decode_codes(q) * np.repeat(dsc, 16, axis=1) * np.float64(a)
    assert np.allclose(d32, ref, rtol=2 ** -23, atol=0)
