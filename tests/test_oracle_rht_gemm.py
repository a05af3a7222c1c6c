"""Pins for the oracle's Hadamard transform, GEMM reference and GELU (CPU)."""
import math

import numpy as np

GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def sylvester16():
    h = np.array([[1]], dtype=np.int64)
    for _ in range(4):
        h = np.block([[h, h], [h, -h]])
    return h


def signs(mask):
    return np.array([-1.0 if (mask >> j) & 1 else 1.0 for j in range(16)])


def test_hadamard_orthogonality_exact():
    h = sylvester16()
    assert np.array_equal(h @ h.T, 16 * np.eye(16, dtype=np.int64))
    # Sylvester order: H[i][j] = (-1)^popcount(i & j)
    for i in range(16):
        for j in range(16):
            assert h[i, j] == (-1) ** bin(i & j).count("1")


def test_rht_block_equals_dense_product(orc):
    h = sylvester16().astype(np.float64)
    rng = np.random.default_rng(0)
    for mask in (0, 0xFFFF, 0xCDAF, 0x1234):
        for _ in range(200):
            x = (rng.standard_normal(16) * 10 ** rng.uniform(-3, 3)).astype(np.float32)
            y = orc.rht16_block(x, mask)
            ref = 0.25 * h @ (signs(mask) * x.astype(np.float64))
            # 4 butterfly stages of fp32 rounding: bound by sum|x|
            bound = 4 * 2 ** -24 * np.abs(x.astype(np.float64)).sum() * 0.25 * 4
            assert np.abs(y - ref).max() <= bound + 1e-45


def test_rht_inverse_and_isometry(orc):
    h = sylvester16().astype(np.float64)
    rng = np.random.default_rng(1)
    mask = 0x5A5A
    x = rng.standard_normal(16).astype(np.float32)
    y = orc.rht16_block(x, mask).astype(np.float64)
    # H is symmetric and H H = 16 I, so x = (1/4) diag(s) H y
    back = 0.25 * signs(mask) * (h @ y)
    assert np.allclose(back, x, rtol=0, atol=1e-6 * np.abs(x).max())
    assert abs(np.dot(y, y) - np.dot(x.astype(np.float64), x)) <= 1e-6 * np.dot(x, x)


def test_rht_preserves_wgrad_product(orc):
    """dY^T X is unchanged when both operands get the same transform along
    the token axis: (H S / 4)^T (H S / 4) = I."""
    rng = np.random.default_rng(2)
    T, A, B = 64, 8, 12
    dy = rng.standard_normal((T, A)).astype(np.float32)
    x = rng.standard_normal((T, B)).astype(np.float32)
    mask = 0xCDAF
    dyt = orc.rht16(dy, 1, mask).astype(np.float64)
    xt = orc.rht16(x, 1, mask).astype(np.float64)
    ref = dy.astype(np.float64).T @ x.astype(np.float64)
    assert np.allclose(dyt.T @ xt, ref, rtol=0, atol=1e-5 * np.abs(ref).max())


def test_rht_axes_are_transposes(orc):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((32, 48)).astype(np.float32)
    a = orc.rht16(x, 1, 0xBEEF)
    b = orc.rht16(np.ascontiguousarray(x.T), 0, 0xBEEF)
    assert np.array_equal(a, b.T)


def test_rht_changes_amax_and_is_used_in_alpha(orc):
    rng = np.random.default_rng(4)
    x = rng.standard_normal((32, 64)).astype(np.float32)
    x[3, 5] = 50.0  # an outlier gets spread over its 16-group
    a_plain = orc.amax(x)
    a_rht = orc.amax(x, rht=True, mask=0xCDAF, block_axis=0)
    assert a_plain == 50.0 and a_rht < 20.0
    _, _, alpha = orc.quantize_1d(x, rht=True, mask=0xCDAF)
    assert alpha == np.float32(np.float32(a_rht) / np.float32(2688.0))


# ------------------------------------------------------------- GEMM
def _random_operand(orc, rows, K, rng, layout):
    x = rng.standard_normal((rows, K)).astype(np.float32)
    c, s, a = orc.quantize_1d(x, sf_layout=layout)
    return (c, s, a, layout)


def _dequant64(orc, op, rows, K):
    """Exact fp64 dequantization written here from the bit fields."""
    c, s, a, layout = op
    c = np.asarray(c, np.uint8)
    q = np.empty((rows, K), np.int64)
    q[:, 0::2] = c & 15
    q[:, 1::2] = c >> 4
    val = np.where(q & 8, -1.0, 1.0) * np.array(GRID)[q & 7]
    out = np.empty((rows, K))
    for r in range(rows):
        for kb in range(K // 16):
            code = int(s[orc.sf_offset(r, kb, K // 16, layout)])
            e, m = code >> 3, code & 7
            d = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
            out[r, kb * 16:(kb + 1) * 16] = val[r, kb * 16:(kb + 1) * 16] * d * float(a)
    return out


def test_gemm_equals_dense_product_of_dequantized(orc):
    rng = np.random.default_rng(5)
    M, N, K = 24, 40, 96
    A = _random_operand(orc, M, K, rng, orc.SF_TCGEN05)
    B = _random_operand(orc, N, K, rng, orc.SF_ROWMAJOR)
    y, s = orc.gemm(A, B, M, N, K)
    ad, bd = _dequant64(orc, A, M, K), _dequant64(orc, B, N, K)
    ref = ad @ bd.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    assert np.allclose(s, np.abs(ad) @ np.abs(bd).T, rtol=1e-12)
    # sampled pairs agree with the full result
    mi = np.array([0, 5, 23, 11]); ni = np.array([39, 0, 17, 3])
    yp, sp = orc.gemm_pairs(A, B, K, mi, ni)
    assert np.array_equal(yp, y[mi, ni]) and np.array_equal(sp, s[mi, ni])


def test_gemm_single_block_is_scalar_product(orc):
    """K = 16 with hand-built codes: Y = alpha_a * alpha_b * d_a * d_b * sum(q_a q_b)."""
    qa = np.array([7, 1, 2, 0, 15, 3, 4, 5, 6, 9, 10, 11, 12, 13, 14, 8], np.uint8)
    qb = np.array([1, 2, 3, 4, 5, 6, 7, 0, 8, 9, 10, 11, 12, 13, 14, 15], np.uint8)
    pack = lambda q: (q[0::2] | (q[1::2] << 4)).astype(np.uint8)[None, :]
    ea, eb = np.array([0x38], np.uint8), np.array([0x41], np.uint8)  # 1.0 and 2.25
    A = (pack(qa), ea, 0.5, 0)
    B = (pack(qb), eb, 3.0, 0)
    y, s = orc.gemm(A, B, 1, 1, 16)
    val = lambda q: (-1 if q & 8 else 1) * GRID[q & 7]
    dot = sum(val(int(a)) * val(int(b)) for a, b in zip(qa, qb))
    assert y[0, 0] == 0.5 * 3.0 * 1.0 * 2.25 * dot
    assert s[0, 0] == 0.5 * 3.0 * 1.0 * 2.25 * sum(abs(val(int(a)) * val(int(b))) for a, b in zip(qa, qb))


def _gelu_tanh_decimal(x: float) -> float:
    """0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))) at 50 significant
    digits with the decimal module: pi from its digits, the square root and
    the exponential from decimal's own correctly rounded routines, tanh from
    the identity tanh(u) = (e^(2u) - 1) / (e^(2u) + 1).  Independent of the
    C library the oracle calls."""
    from decimal import Decimal, getcontext
    getcontext().prec = 50
    pi = Decimal("3.14159265358979323846264338327950288419716939937510")
    X = Decimal(x)
    u = (Decimal(2) / pi).sqrt() * (X + Decimal("0.044715") * X * X * X)
    e = (2 * u).exp()
    return float(Decimal("0.5") * X * (1 + (e - 1) / (e + 1)))


def test_gelu_tanh_against_an_independent_evaluation(orc):
    """The tanh-form GELU at points spanning its curved range and tails,
    within a few double ulps of max(|GELU(x)|, |x|) of the 50-digit
    evaluation (in the negative tail 1 + tanh(u) cancels, so the double
    formula is accurate to |x| ulps there, not to GELU's own): a coefficient
    off in its fourth digit, a dropped cubic term or a sign error fails by
    orders of magnitude more."""
    for x in [-8.0, -5.5, -3.0, -2.25, -1.0, -0.5, -0.125, 1e-6, 0.25, 0.7, 1.0, 1.5, 2.0,
              3.25, 4.5, 7.0]:
        want = _gelu_tanh_decimal(x)
        got = orc.gelu_tanh(x)
        assert abs(got - want) <= 4e-16 * max(abs(want), abs(x)), (x, got, want)


def test_gelu_tanh(orc):
    assert orc.gelu_tanh(0.0) == 0.0
    for x in np.linspace(-6, 6, 61):
        g, gm = orc.gelu_tanh(x), orc.gelu_tanh(-x)
        assert abs((g - gm) - x) < 1e-12  # gelu(x) - gelu(-x) = x
        exact = 0.5 * x * (1 + math.erf(x / math.sqrt(2)))
        assert abs(g - exact) < 1e-3  # tanh form approximates x*Phi(x)
