"""Pins for the oracle's LoRA branch of a W4A4 linear layer (notes, §3.4
"NVFP4 training and DMD LoRA": quantized backbone weight plus a bf16
rank-r adapter, scale = alpha / rank).  Checked against what the pages'
definition and linear algebra fix, not against a retyped sum: the merged
form x (scale B A)^T of the pages' W ~ Dequant(Q(W0)) + delta W equals the
branch computed from u = x A^T; closed forms for zero, rank-1 and identity
adapters; scale linearity; and the tolerance scale's bound."""
import numpy as np
import pytest

from nvfp4_block_scaled_20_b200 import synth


def _rand(seed, *shape):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape).astype(np.float32)


def test_merged_weight_form_equals_the_factored_branch(orc):
    """x (B A)^T * scale (the adapter merged into the weight, the pages'
    W + delta W) equals scale * (x A^T) B^T from u = x A^T: associativity of
    the product, within fp64 rounding."""
    M, N, Kin, r = 24, 40, 64, 8
    x = _rand(1, M, Kin).astype(np.float64)
    a = _rand(2, r, Kin).astype(np.float64)
    b = _rand(3, N, r).astype(np.float64)
    scale = 128.0 / 8
    merged = x @ (scale * (b @ a)).T
    u = (x @ a.T).astype(np.float32)  # exact only to fp32: compare with that u
    y0 = np.zeros((M, N))
    y, s = orc.lora_add(y0, y0, u, b.astype(np.float32), scale)
    ref = u.astype(np.float64) @ b.T * scale
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-9)
    assert np.allclose(y, merged, rtol=1e-5, atol=1e-3)  # u rounded to fp32
    assert (s >= np.abs(y) - 1e-9).all()


def test_zero_rank_one_and_identity_adapters(orc):
    M, N, r = 5, 7, 3
    base_y = _rand(4, M, N).astype(np.float64)
    base_s = np.abs(base_y)
    u = _rand(5, M, r)
    # B = 0: the branch adds nothing
    y, s = orc.lora_add(base_y, base_s, u, np.zeros((N, r), np.float32), 2.0)
    assert np.array_equal(y, base_y) and np.array_equal(s, base_s)
    # rank 1 with u = 1: every row gains scale * v
    v = _rand(6, N)
    u1 = np.zeros((M, 1), np.float32) + 1.0
    y, s = orc.lora_add(base_y, base_s, u1, v[:, None], -0.5)
    assert np.array_equal(y, base_y + (-0.5) * v.astype(np.float64)[None, :])
    assert np.array_equal(s, base_s + 0.5 * np.abs(v.astype(np.float64))[None, :])
    # B = I (r = N): the branch is scale * u itself
    ui = _rand(7, M, N)
    y, _ = orc.lora_add(np.zeros((M, N)), np.zeros((M, N)), ui, np.eye(N, dtype=np.float32), 3.0)
    assert np.array_equal(y, 3.0 * ui.astype(np.float64))


def test_scale_linearity_and_shape_check(orc):
    M, N, r = 6, 10, 4
    u, b = _rand(8, M, r), _rand(9, N, r)
    z = np.zeros((M, N))
    y1, _ = orc.lora_add(z, z, u, b, 1.0)
    y2, _ = orc.lora_add(z, z, u, b, 2.0)
    assert np.array_equal(y2, 2.0 * y1)  # power-of-two scale: exact
    with pytest.raises(ValueError):
        orc.lora_add(z, z, u, b[:, :3], 1.0)


def test_on_a_w4a4_base(orc):
    """The branch adds to the oracle's W4A4 output: with a zero adapter the
    layer output is the base GEMM, with a nonzero one it moves by exactly the
    branch (the base is not recomputed)."""
    x, w = synth.tiny_linear()
    aq = orc.quantize_1d(x.numpy(), sf_layout=orc.SF_TCGEN05)
    bq = orc.quantize_2d(w.numpy(), sf_layout=orc.SF_TCGEN05)
    y, s = orc.gemm((aq[0], aq[1], aq[2], 1), (bq[0], bq[1], bq[2], 1), 64, 128, 256)
    u = _rand(10, 64, 16)
    b = _rand(11, 128, 16)
    yl, sl = orc.lora_add(y, s, u, b, 1.0)
    delta, _ = orc.lora_add(np.zeros_like(y), np.zeros_like(s), u, b, 1.0)
    assert np.allclose(yl - y, delta, rtol=0, atol=1e-12 * (np.abs(y).max() + np.abs(delta).max()))
    assert (sl >= s).all()
