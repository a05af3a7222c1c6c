"""GPU parity of the quantizers, RHT and dequantizer against the oracle:
bit-exact codes, scale bytes (including tcgen05 padding) and global scales,
on seeded inputs spanning several 128-row scale atoms and ragged tails."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_block_scaled_20_b200 as nv
from nvfp4_block_scaled_20_b200 import synth
from gpu_helpers import DEV, assert_q_equal, mismatch_report, require_gpu, to_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


LAYOUTS = [nv.NVFP4_SF_ROWMAJOR, nv.NVFP4_SF_TCGEN05]


# ------------------------------------------------------------ conversions
def test_e2m1_rounding_through_quantizer():
    """Blocks led by 6.0 with alpha pinned to 1 have scale exactly 1, so every
    other element is encoded as round-to-E2M1(y): sweeps every tie of the
    element grid +-8 ulp, plus random values, against the oracle."""
    vals = []
    for m in [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0]:
        b = np.float32(m).view(np.uint32)
        vals.append((np.arange(-8, 9, dtype=np.int64) + b).astype(np.uint32).view(np.float32))
    rng = np.random.default_rng(0)
    vals.append(rng.uniform(-6, 6, 200000).astype(np.float32))
    vals.append(np.array([0.0, -0.0, 1e-30, -1e-30, 5.999, -5.999], np.float32))
    v = np.concatenate(vals)
    v = np.concatenate([v, -v])
    nb = (v.size + 14) // 15
    x = np.zeros((nb, 16), np.float32)
    x[:, 0] = 6.0
    flat = np.zeros(nb * 15, np.float32)
    flat[: v.size] = v
    x[:, 1:] = flat.reshape(nb, 15)
    rows = ((nb + 15) // 16) * 16
    xx = np.zeros((rows, 16), np.float32)
    xx[:nb] = x
    xx[nb:, 0] = 6.0
    alpha = torch.ones(1, device=DEV)
    q = nv.quantize_1d(torch.from_numpy(xx).to(DEV), four_over_six=False, alpha_in=alpha,
                       sf_layout=nv.NVFP4_SF_ROWMAJOR)
    ref = oracle.quantize_1d(xx, four_over_six=False, alpha_in=1.0, sf_layout=oracle.SF_ROWMAJOR)
    assert (ref[1] == 0x38).all()  # scale 1.0
    assert_q_equal(q, ref, "e2m1 sweep")


def test_e4m3_rounding_through_quantizer():
    """Block maxima sweeping the E4M3 grid (every midpoint +-4 ulp and random
    values from 2^-12 to 2^10 times 6) with alpha = 1: the scale byte is the
    E4M3 rounding of bmax / 6."""
    tab = [oracle.e4m3_decode(c) for c in range(0x7F)]
    ts = []
    for i in range(len(tab) - 1):
        mid = np.float32((tab[i] + tab[i + 1]) / 2).view(np.uint32)
        ts.append((np.arange(-4, 5, dtype=np.int64) + mid).astype(np.uint32).view(np.float32))
    rng = np.random.default_rng(1)
    ts.append((2.0 ** rng.uniform(-12, 10, 40000)).astype(np.float32))
    t = np.concatenate(ts)
    bmax = (t.astype(np.float64) * 6).astype(np.float32)
    n = ((t.size + 15) // 16) * 16
    x = np.zeros((n, 16), np.float32)
    x[: t.size, 3] = bmax
    x[: t.size, 7] = -bmax * np.float32(0.3)
    alpha = torch.ones(1, device=DEV)
    for fos in (False, True):
        q = nv.quantize_1d(torch.from_numpy(x).to(DEV), four_over_six=fos, alpha_in=alpha,
                           sf_layout=nv.NVFP4_SF_ROWMAJOR)
        ref = oracle.quantize_1d(x, four_over_six=fos, alpha_in=1.0, sf_layout=oracle.SF_ROWMAJOR)
        assert_q_equal(q, ref, "e4m3 sweep fos=%d" % fos)


# ------------------------------------------------------------ 1D
@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("fos", [True, False])
def test_quantize_1d_bf16_activation(layout, fos):
    x = synth.activation(1, 11, 300, 3072)  # 2 full 128-row bands + ragged 44 rows
    q = nv.quantize_1d(x.to(DEV), four_over_six=fos, sf_layout=layout)
    ref = oracle.quantize_1d(to_oracle(x), four_over_six=fos, sf_layout=layout)
    assert_q_equal(q, ref, "1d bf16")


def test_quantize_1d_fp32_tiny_linear():
    x, w = synth.tiny_linear()
    for layout in LAYOUTS:
        q = nv.quantize_1d(x.to(DEV), sf_layout=layout)
        assert_q_equal(q, oracle.quantize_1d(to_oracle(x), sf_layout=layout), "tiny X")


def test_quantize_1d_strided_rows_and_ragged_blocks():
    base = synth.activation(5, 1, 130, 256 + 32, n_out=3)  # ld = 288, cols used = 208
    x = base[:, :208]
    q = nv.quantize_1d(base.to(DEV)[:, :208], sf_layout=1)
    ref = oracle.quantize_1d(to_oracle(x), sf_layout=oracle.SF_TCGEN05)
    assert_q_equal(q, ref, "strided")


def test_quantize_1d_global_scale_in_and_global_scale_call():
    x = synth.activation(6, 1, 256, 512)
    xd = x.to(DEV)
    a = nv.global_scale(xd)
    ref_alpha = oracle.quantize_1d(to_oracle(x))[2]
    assert float(a.cpu()[0]) == np.float32(ref_alpha)
    a2 = torch.full((1,), 0.01, device=DEV)
    q = nv.quantize_1d(xd, alpha_in=a2)
    ref = oracle.quantize_1d(to_oracle(x), alpha_in=0.01, sf_layout=oracle.SF_TCGEN05)
    assert_q_equal(q, ref, "alpha_in")


def test_quantize_edge_cases():
    # all zero -> alpha 1, zero codes and scales
    z = torch.zeros(64, 64, dtype=torch.bfloat16)
    assert_q_equal(nv.quantize_1d(z.to(DEV)), oracle.quantize_1d(to_oracle(z), sf_layout=1), "zeros")
    # constant, tiny (subnormal scales) and huge magnitudes, mixed
    x = torch.zeros(48, 128)
    x[0:16] = 3.3
    x[16:32] = torch.linspace(-1e-6, 1e-6, 16 * 128).reshape(16, 128)
    x[32:48] = torch.linspace(-3e30, 3e30, 16 * 128).reshape(16, 128)
    x[40, 5] = 0.0
    for dt in (torch.float32, torch.bfloat16):
        xx = x.to(dt)
        assert_q_equal(nv.quantize_1d(xx.to(DEV)), oracle.quantize_1d(to_oracle(xx), sf_layout=1),
                       "edge %s" % dt)
    # blocks whose scale rounds to zero relative to a huge tensor max
    y = torch.full((16, 32), 1e-12)
    y[0, 0] = 1e6
    assert_q_equal(nv.quantize_1d(y.to(DEV)), oracle.quantize_1d(to_oracle(y), sf_layout=1), "zero-scale")


def test_quantize_empty_is_noop():
    x = torch.zeros(0, 64, device=DEV)
    q = nv.quantize_1d(x)
    assert q.codes.numel() == 0


# ------------------------------------------------------------ 2D
@pytest.mark.parametrize("layout", LAYOUTS)
def test_quantize_2d_weight(layout):
    w = synth.weight(1, 12, 272, 3072)  # 2 bands + 16 ragged rows
    q = nv.quantize_2d(w.to(DEV), sf_layout=layout)
    assert_q_equal(q, oracle.quantize_2d(to_oracle(w), sf_layout=layout), "2d")


def test_quantize_2d_odd_tile_count_and_fp32():
    x, w = synth.tiny_linear()
    assert_q_equal(nv.quantize_2d(w.to(DEV)), oracle.quantize_2d(to_oracle(w), sf_layout=1), "tiny W")
    w2 = synth.weight(3, 3, 48, 16 * 7, dtype=torch.float32)  # 7 tiles per band: odd
    assert_q_equal(nv.quantize_2d(w2.to(DEV)), oracle.quantize_2d(to_oracle(w2), sf_layout=1), "odd")
    for fos in (True, False):
        assert_q_equal(nv.quantize_2d(w2.to(DEV), four_over_six=fos),
                       oracle.quantize_2d(to_oracle(w2), four_over_six=fos, sf_layout=1), "fos")


# ------------------------------------------------------------ mixed 1D + 2D launch
@pytest.mark.parametrize("layout", LAYOUTS)
def test_quantize_mixed_matches_oracle(layout):
    """1D activations (ragged rows, outlier channels, a strided view) and 2D
    weights in one mixed call: every tensor bit-exact with the oracle's 1D /
    2D quantization under its own global scale."""
    x = synth.activation(21, 2, 300, 3072)
    w = synth.weight(22, 3, 272, 3072)
    base = synth.activation(23, 1, 130, 288, n_out=3)
    w_small = synth.weight(24, 4, 48, 16 * 7, dtype=torch.bfloat16)  # odd tile count per band
    xs = [x.to(DEV), w.to(DEV), base.to(DEV)[:, :208], w_small.to(DEV)]
    flags = [False, True, False, True]
    qs = nv.quantize_mixed(xs, flags, sf_layout=layout)
    refs = [oracle.quantize_1d(to_oracle(x), sf_layout=layout),
            oracle.quantize_2d(to_oracle(w), sf_layout=layout),
            oracle.quantize_1d(to_oracle(base[:, :208]), sf_layout=layout),
            oracle.quantize_2d(to_oracle(w_small), sf_layout=layout)]
    for i, (q, ref) in enumerate(zip(qs, refs)):
        assert_q_equal(q, ref, "mixed[%d]" % i)


def test_quantize_mixed_qkv_shapes_equal_single_calls():
    """The DiT QKV operands (X [2640, 3072] 1D, W [9216, 3072] 2D) through one
    mixed call equal the separate quantize_1d / quantize_2d calls byte for
    byte (those are pinned to the oracle above and at full size elsewhere),
    and sampled rows equal the oracle directly; plus an fp32 pair and an
    empty tensor (global scale 1, nothing else written)."""
    x, w = synth.qkv_linear(DEV)
    qs = nv.quantize_mixed([x, w], [False, True])
    q1 = nv.quantize_1d(x)
    q2 = nv.quantize_2d(w)
    for a, b, what in ((qs[0], q1, "X"), (qs[1], q2, "W")):
        assert torch.equal(a.codes, b.codes), what
        assert torch.equal(a.scales, b.scales), what
        assert torch.equal(a.alpha, b.alpha), what
    # oracle on a band of each (alpha from the full tensor)
    xa, wa = float(q1.alpha.cpu()[0]), float(q2.alpha.cpu()[0])
    xr = to_oracle(x[256:384].cpu())
    ref = oracle.quantize_1d(xr, alpha_in=xa, sf_layout=oracle.SF_ROWMAJOR)
    assert np.array_equal(qs[0].codes[256:384].cpu().numpy(), ref[0])
    wr = to_oracle(w[512:640].cpu())
    ref = oracle.quantize_2d(wr, alpha_in=wa, sf_layout=oracle.SF_ROWMAJOR)
    assert np.array_equal(qs[1].codes[512:640].cpu().numpy(), ref[0])
    # fp32 inputs and an empty tensor in the batch
    a32 = synth.activation(25, 1, 64, 256).float().to(DEV)
    w32 = synth.weight(26, 1, 64, 256, dtype=torch.float32).to(DEV)
    empty = torch.zeros(0, 256, device=DEV)
    qs = nv.quantize_mixed([a32, empty, w32], [False, False, True])
    assert_q_equal(qs[0], oracle.quantize_1d(to_oracle(a32.cpu()), sf_layout=1), "fp32 1d")
    assert_q_equal(qs[2], oracle.quantize_2d(to_oracle(w32.cpu()), sf_layout=1), "fp32 2d")
    assert float(qs[1].alpha.cpu()[0]) == 1.0


# ------------------------------------------------------------ RHT / transposed
def test_rht16_standalone_both_axes():
    mask = synth.rht_sign_mask(0)
    x = synth.activation(4, 2, 96, 160)
    for axis in (0, 1):
        got = nv.rht16(x.to(DEV), block_axis=axis, mask=mask).cpu().numpy()
        want = oracle.rht16(to_oracle(x), axis, mask)
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), mismatch_report(got, want, "rht")


@pytest.mark.parametrize("rht", [True, False])
@pytest.mark.parametrize("layout", LAYOUTS)
def test_quantize_transposed(rht, layout):
    """WGRAD operand path: 16-blocks along tokens, RHT fused, output K-major.
    1040 tokens = 16 full 64-row chunks + one 16-row chunk; 200 features."""
    mask = synth.rht_sign_mask(0)
    dy = synth.activation(4, 1, 1040, 200, n_out=0, std=1e-3)
    x = synth.activation(4, 2, 1040, 200)
    for t in (dy, x):
        q = nv.quantize_1d(t.to(DEV), rht=rht, mask=mask, block_axis=1, sf_layout=layout)
        ref = oracle.quantize_1d(to_oracle(t), rht=rht, mask=mask, block_axis=1, sf_layout=layout)
        assert_q_equal(q, ref, "transposed rht=%d" % rht)
        a = nv.global_scale(t.to(DEV), rht=rht, mask=mask, block_axis=1)
        assert float(a.cpu()[0]) == np.float32(ref[2])


def test_quantize_transposed_strided_batched_and_fp32():
    """The row-axis path on a strided bf16 input (row stride 264 > 200
    columns), two bf16 tensors of different shapes in one batched call, and
    an fp32 input, each against the oracle."""
    from nvfp4_block_scaled_20_b200 import capi
    mask = synth.rht_sign_mask(0)
    base = synth.activation(4, 3, 336, 264)
    x = base[:, :200]
    q = nv.quantize_1d(base.to(DEV)[:, :200], rht=True, mask=mask, block_axis=1)
    assert_q_equal(q, oracle.quantize_1d(to_oracle(x), rht=True, mask=mask, block_axis=1,
                                         sf_layout=1), "strided")
    xs = [synth.activation(4, 5, 1040, 136).to(DEV), synth.activation(4, 6, 208, 384).to(DEV)]
    outs = [nv.QTensor(*nv._alloc_q(t.shape[1], t.shape[0], 1, DEV), t.shape[1], t.shape[0], 1)
            for t in xs]
    ws = nv.workspace(2)
    d = (capi.nvfp4_tensor_desc * 2)()
    for i, (t, o) in enumerate(zip(xs, outs)):
        d[i] = capi.nvfp4_tensor_desc(t.data_ptr(), None, o.codes.data_ptr(), o.scales.data_ptr(),
                                      o.alpha.data_ptr(), t.shape[0], t.shape[1], t.stride(0))
    qp = capi.nvfp4_qparams(1, 1, mask, 1, 1, 0, None)
    st = capi.nvfp4_quantize_1d_batched(d, 2, capi.NVFP4_BF16, qp, ws.data_ptr(), ws.numel(),
                                        torch.cuda.current_stream().cuda_stream)
    assert st == 0
    for t, o in zip(xs, outs):
        assert_q_equal(o, oracle.quantize_1d(to_oracle(t), rht=True, mask=mask, block_axis=1,
                                             sf_layout=1), "batched")
    xf = synth.activation(4, 7, 272, 96, dtype=torch.float32)
    q = nv.quantize_1d(xf.to(DEV), rht=True, mask=mask, block_axis=1)
    assert_q_equal(q, oracle.quantize_1d(xf.numpy(), rht=True, mask=mask, block_axis=1,
                                         sf_layout=1), "fp32")


def test_quantize_rht_rows():
    mask = 0x1234
    x = synth.activation(7, 1, 144, 320)
    q = nv.quantize_1d(x.to(DEV), rht=True, mask=mask)
    assert_q_equal(q, oracle.quantize_1d(to_oracle(x), rht=True, mask=mask, sf_layout=1), "rht rows")


# ------------------------------------------------------------ KV batched + dequant
def test_kv_batched_quantize_and_dequant():
    ts = [synth.kv_tensor(3, l, w, heads=24, tokens=40) for l in range(3) for w in range(2)]
    qs = nv.quantize_1d_batched([t.to(DEV) for t in ts])
    for t, q in zip(ts, qs):
        ref = oracle.quantize_1d(to_oracle(t), sf_layout=oracle.SF_ROWMAJOR)
        assert_q_equal(q, ref, "kv")
    outs = nv.dequantize(qs)
    outs32 = nv.dequantize(qs, out_dtype=torch.float32)
    for t, q, o, o32 in zip(ts, qs, outs, outs32):
        ref = oracle.quantize_1d(to_oracle(t), sf_layout=oracle.SF_ROWMAJOR)
        d32, d16 = oracle.dequantize(ref[0], ref[1], ref[2], t.shape[0], t.shape[1])
        g16 = o.cpu().view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(g16, d16), mismatch_report(g16, d16, "dequant bf16")
        g32 = o32.cpu().numpy()
        assert np.array_equal(g32.view(np.uint32), d32.view(np.uint32))


def test_dequant_tcgen05_layout():
    w = synth.weight(8, 1, 160, 512)
    q = nv.quantize_2d(w.to(DEV))
    out = nv.dequantize([q], out_dtype=torch.float32)[0].cpu().numpy()
    ref = oracle.quantize_2d(to_oracle(w), sf_layout=oracle.SF_TCGEN05)
    d32, _ = oracle.dequantize(ref[0], ref[1], ref[2], 160, 512, oracle.SF_TCGEN05)
    assert np.array_equal(out.view(np.uint32), d32.view(np.uint32))


@pytest.mark.parametrize("layout", [nv.NVFP4_SF_ROWMAJOR, nv.NVFP4_SF_TCGEN05])
def test_window_gather_dequant(layout):
    """Global sink, shot sink (START, LEN) and recent window of every head,
    overlapping and touching ranges included, against the oracle's dequant
    of the union of those rows (in row order), bit for bit."""
    heads, tokens = 6, 300
    ts = [synth.kv_tensor(3, l, w, heads=heads, tokens=tokens) for l in range(2) for w in range(2)]
    qs = nv.quantize_1d_batched([t.to(DEV) for t in ts], sf_layout=layout)
    token_ranges = [(0, 8), (100, 108), (104, 112), (112, 120), (250, 300), (299, 300), (7, 7)]
    ranges = nv.window_row_ranges(heads, tokens, token_ranges)
    rows = sorted({r for b, e in ranges for r in range(b, e)})
    for dt in (torch.bfloat16, torch.float32):
        outs = nv.dequantize_rows(qs, ranges, out_dtype=dt)
        for t, q, o in zip(ts, qs, outs):
            assert o.shape[0] == len(rows)
            ref = oracle.quantize_1d(to_oracle(t), sf_layout=layout)
            d32, d16 = oracle.dequantize(ref[0], ref[1], ref[2], t.shape[0], t.shape[1], layout)
            if dt == torch.bfloat16:
                got = o.cpu().view(torch.int16).numpy().view(np.uint16)
                want = d16[rows]
            else:
                got = o.cpu().numpy().view(np.uint32)
                want = d32[rows].view(np.uint32)
            assert np.array_equal(got, want), mismatch_report(got, want, "gather dequant")


@pytest.mark.parametrize("rows,cols", [(144, 176), (160, 272), (64, 64)])
@pytest.mark.parametrize("lin,lout", [(nv.NVFP4_SF_ROWMAJOR, nv.NVFP4_SF_ROWMAJOR),
                                      (nv.NVFP4_SF_TCGEN05, nv.NVFP4_SF_TCGEN05),
                                      (nv.NVFP4_SF_TCGEN05, nv.NVFP4_SF_ROWMAJOR)])
def test_transpose_2d(rows, cols, lin, lout):
    """The weight operand of the data-gradient GEMM: the transposed 2D
    encoding, codes and scale bytes (padding included) bit for bit."""
    w = synth.weight(12, 1, rows, cols)
    q = nv.quantize_2d(w.to(DEV), sf_layout=lin)
    t = nv.transpose_2d(q, sf_layout=lout)
    ref = oracle.quantize_2d(to_oracle(w), sf_layout=lin)
    assert_q_equal(q, ref, "W")
    tc, ts = oracle.transpose_2d(ref[0], ref[1], rows, cols, lin, lout)
    assert (t.rows, t.cols) == (cols, rows)
    assert_q_equal(t, (tc, ts, ref[2]), "W^T")
