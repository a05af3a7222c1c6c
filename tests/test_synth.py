"""The seeded input generator: counter-based splitmix64 against a pure-Python
restatement, determinism, and the recipes' shapes and structure (CPU)."""
import math

import numpy as np
import torch

from nvfp4_block_scaled_20_b200 import synth


def _py_splitmix(seed, sid, i):
    key = synth.stream_key(seed, sid)
    return synth.mix64_int((key + i * synth.GAMMA) & synth.MASK64)


def test_splitmix_matches_python_ints():
    r = synth.raw64(3, 7, 1000, 64)
    for j in range(64):
        want = _py_splitmix(3, 7, 1000 + j)
        got = int(r[j]) & synth.MASK64
        assert got == want


def test_splitmix_reference_vector():
    # splitmix64 seeded with 0: first output 0xE220A8397B1DCDAF (public test vector)
    assert synth.mix64_int(0 + synth.GAMMA) == 0xE220A8397B1DCDAF
    assert synth.rht_sign_mask(0) == 0xCDAF


def test_uniform_and_normal_moments():
    u = synth.uniform(0, 1, 200000)
    assert 0 < float(u.min()) and float(u.max()) < 1
    assert abs(float(u.mean()) - 0.5) < 0.005
    z = synth.normal(0, 2, 200001)
    assert z.numel() == 200001
    assert abs(float(z.mean())) < 0.01 and abs(float(z.std()) - 1) < 0.01


def test_deterministic_and_streams_differ():
    a = synth.normal(5, 1, 1000)
    b = synth.normal(5, 1, 1000)
    c = synth.normal(5, 2, 1000)
    assert torch.equal(a, b) and not torch.equal(a, c)


def test_activation_recipe_structure():
    x = synth.activation(1, 1, 256, 3072)
    assert x.dtype == torch.bfloat16 and x.shape == (256, 3072)
    cols = synth.choose_columns(1, 1 + 0x5000, 3072, 31)
    assert len(set(cols)) == 31
    colmax = x.float().abs().amax(dim=0)
    others = torch.ones(3072, dtype=torch.bool)
    others[cols] = False
    # heavy-tailed (Student-t x 8) columns dominate the Gaussian ones
    assert float(colmax[cols].median()) > 3 * float(colmax[others].median())


def test_tiny_recipe():
    x, w = synth.tiny_linear()
    assert x.shape == (64, 256) and w.shape == (128, 256)
    assert x.dtype == torch.float32
    assert abs(float(w.std()) - 0.02) < 0.002


def test_kv_recipe_bias_per_head():
    kv = synth.kv_tensor(3, 0, 0, heads=4, tokens=256, head_dim=128)
    assert kv.shape == (4 * 256, 128) and kv.dtype == torch.bfloat16
    means = kv.float().reshape(4, -1).mean(dim=1)
    bias = synth.normal(3, 0x100 + 0x8000, 4) * 2.0
    assert torch.allclose(means.double(), bias, atol=0.05)


def test_activation_cols_is_a_column_slice_of_activation():
    from nvfp4_block_scaled_20_b200 import synth
    full = synth.activation(4, 2, 96, 1440)  # 15 outlier columns
    for c0, c1 in ((0, 64), (96, 352), (1376, 1440)):
        part = synth.activation_cols(4, 2, 96, 1440, c0, c1)
        assert torch.equal(part, full[:, c0:c1]), (c0, c1)
    full = synth.activation(4, 1, 64, 320, n_out=0, std=1e-3)
    assert torch.equal(synth.activation_cols(4, 1, 64, 320, 32, 96, n_out=0, std=1e-3),
                       full[:, 32:96])
