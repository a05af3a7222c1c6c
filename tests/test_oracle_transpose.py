"""Pins for the oracle's transpose of a 2D (16x16-tile) encoding, the operand
of the data-gradient GEMM ("The three GEMMs of backpropagation in NVFP4":
DGRAD takes the weight in NVFP4; 2D block scaling for weights).  Checked
against properties that do not reuse the function's index arithmetic: a
double transpose is the identity, dequantizing the transpose equals
transposing the dequantized matrix (values, through the separately pinned
dequantizer, in both scale layouts), and a fresh 2D quantization of W^T
agrees on every tile but near-ties of the 4-vs-6 pick (its tile error is
summed in the other order)."""
import numpy as np
import pytest

from nvfp4_block_scaled_20_b200 import synth


def _w(rows, cols, seed=6):
    return synth.weight(seed, 1, rows, cols).float().numpy()


@pytest.mark.parametrize("rows,cols", [(16, 16), (48, 96), (160, 272)])
def test_double_transpose_is_identity(orc, rows, cols):
    codes, scales, alpha = orc.quantize_2d(_w(rows, cols))
    tc, ts = orc.transpose_2d(codes, scales, rows, cols)
    assert tc.shape == (cols, rows // 2)
    bc, bs = orc.transpose_2d(tc, ts, cols, rows)
    assert np.array_equal(bc, codes)
    assert np.array_equal(bs, scales)


@pytest.mark.parametrize("lin,lout", [(0, 0), (0, 1), (1, 0), (1, 1)])
def test_dequant_of_transpose_is_transpose_of_dequant(orc, lin, lout):
    rows, cols = 144, 176  # ragged against the 128-row atoms of the tcgen05 layout
    codes, scales, alpha = orc.quantize_2d(_w(rows, cols, 7), sf_layout=lin)
    tc, ts = orc.transpose_2d(codes, scales, rows, cols, lin, lout)
    d, _ = orc.dequantize(codes, scales, alpha, rows, cols, lin)
    dt, _ = orc.dequantize(tc, ts, alpha, cols, rows, lout)
    assert np.array_equal(dt.view(np.uint32), np.ascontiguousarray(d.T).view(np.uint32))


def test_agrees_with_quantizing_the_transpose(orc):
    rows, cols = 256, 512
    w = _w(rows, cols, 8)
    codes, scales, alpha = orc.quantize_2d(w)
    tc, ts = orc.transpose_2d(codes, scales, rows, cols)
    fc, fs, falpha = orc.quantize_2d(np.ascontiguousarray(w.T), alpha_in=alpha)
    assert falpha == alpha
    tiles = 0
    bad = 0
    for tr in range(cols // 16):
        for tcb in range(rows // 16):
            tiles += 1
            a = tc[tr * 16:(tr + 1) * 16, tcb * 8:(tcb + 1) * 8]
            b = fc[tr * 16:(tr + 1) * 16, tcb * 8:(tcb + 1) * 8]
            sa = ts.reshape(cols, rows // 16)[tr * 16, tcb]
            sb = fs.reshape(cols, rows // 16)[tr * 16, tcb]
            if not (np.array_equal(a, b) and sa == sb):
                bad += 1
    # a different summation order can only flip near-tied picks
    assert bad <= tiles // 200, (bad, tiles)


def test_bad_shape(orc):
    codes, scales, _ = orc.quantize_2d(_w(32, 32))
    with pytest.raises(ValueError):
        orc.transpose_2d(codes, scales, 32, 24)
