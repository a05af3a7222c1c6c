"""GPU parity of the tcgen05 block-scaled FP4 GEMM against the oracle's fp64
GEMM on the same encodings: |gpu - oracle| <= 1e-3 * sum_k |a_k b_k| (plus
half a bf16 ulp of the reference for bf16 outputs), on shapes that span
several tiles, ragged M / N tails, partial K stages and both tile widths."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_block_scaled_20_b200 as nv
from nvfp4_block_scaled_20_b200 import capi, synth
from gpu_helpers import (DEV, assert_q_equal, gemm_tolerance, oracle_gemm_ref, require_gpu,
                         to_oracle)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def upload(ref, rows, cols):
    """Oracle encoding -> device QTensor (tcgen05 scale layout)."""
    codes, scales, alpha = ref
    return nv.QTensor(torch.from_numpy(codes).to(DEV), torch.from_numpy(scales).to(DEV),
                      torch.tensor([alpha], dtype=torch.float32, device=DEV), rows, cols,
                      nv.NVFP4_SF_TCGEN05)


def run_case(x, w, out_dtype, epilogue=nv.NVFP4_EPI_NONE, x2d=False):
    M, K = x.shape
    N = w.shape[0]
    aref = (oracle.quantize_2d if x2d else oracle.quantize_1d)(to_oracle(x), sf_layout=oracle.SF_TCGEN05)
    bref = oracle.quantize_2d(to_oracle(w), sf_layout=oracle.SF_TCGEN05)
    ws = nv.workspace(0)
    out = nv.gemm(upload(aref, M, K), upload(bref, N, K), out_dtype=out_dtype, epilogue=epilogue,
                  ws=ws)
    assert nv.device_error(ws) == 0
    y, s = oracle_gemm_ref(aref, bref, M, N, K)
    if epilogue == nv.NVFP4_EPI_GELU_TANH:
        y = np.vectorize(oracle.gelu_tanh)(y)
    got = out.float().cpu().numpy().astype(np.float64)
    tol = gemm_tolerance(y, s, out_dtype == torch.bfloat16, epilogue == nv.NVFP4_EPI_GELU_TANH)
    err = np.abs(got - y)
    bad = np.argwhere(err > tol)
    assert bad.size == 0, "%d outputs out of tolerance, first %s: gpu=%r ref=%r tol=%r" % (
        len(bad), bad[0], got[tuple(bad[0])], y[tuple(bad[0])], tol[tuple(bad[0])])
    return got, y, s


def test_tiny_linear_fp32_and_bf16():
    x, w = synth.tiny_linear()  # M=64, N=128, K=256: one tile, BN=128 path
    for dt in (torch.float32, torch.bfloat16):
        run_case(x, w, dt)


@pytest.mark.parametrize("M,N,K", [(200, 272, 320), (128, 256, 4096), (300, 384, 576),
                                   (64, 128, 64), (1, 16, 256), (257, 512, 3072)])
def test_shapes_bf16_inputs(M, N, K):
    x = synth.activation(9, M + N, M, K)
    w = synth.weight(9, K, N, K)
    run_case(x, w, torch.float32)
    run_case(x, w, torch.bfloat16)


def test_gelu_epilogue():
    x = synth.activation(10, 1, 130, 512)
    w = synth.weight(10, 2, 256, 512)
    run_case(x, w, torch.bfloat16, nv.NVFP4_EPI_GELU_TANH)
    run_case(x, w, torch.float32, nv.NVFP4_EPI_GELU_TANH)


def test_gpu_quantized_operands_end_to_end():
    """The quantizers' device outputs fed straight into the GEMM (the product
    path), codes checked bit-exact and the product within tolerance."""
    x = synth.activation(11, 1, 192, 768)
    w = synth.weight(11, 2, 320, 768)
    qa = nv.quantize_1d(x.to(DEV))
    qb = nv.quantize_2d(w.to(DEV))
    aref = oracle.quantize_1d(to_oracle(x), sf_layout=1)
    bref = oracle.quantize_2d(to_oracle(w), sf_layout=1)
    assert_q_equal(qa, aref, "A")
    assert_q_equal(qb, bref, "B")
    out = nv.gemm(qa, qb, out_dtype=torch.float32).cpu().numpy()
    y, s = oracle_gemm_ref(aref, bref, 192, 320, 768)
    assert (np.abs(out - y) <= gemm_tolerance(y, s, False)).all()


def test_wgrad_shape_transposed_operands():
    """dW = dY^T X with both operands RHT-transformed and quantized along the
    tokens (K), fp32 output."""
    mask = synth.rht_sign_mask(0)
    dy = synth.activation(4, 1, 1024, 128, n_out=0, std=1e-3)
    x = synth.activation(4, 2, 1024, 272)
    qa = nv.quantize_1d(dy.to(DEV), rht=True, mask=mask, block_axis=1)
    qb = nv.quantize_1d(x.to(DEV), rht=True, mask=mask, block_axis=1)
    aref = oracle.quantize_1d(to_oracle(dy), rht=True, mask=mask, block_axis=1, sf_layout=1)
    bref = oracle.quantize_1d(to_oracle(x), rht=True, mask=mask, block_axis=1, sf_layout=1)
    assert_q_equal(qa, aref, "dY^T")
    assert_q_equal(qb, bref, "X^T")
    out = nv.gemm(qa, qb, out_dtype=torch.float32).cpu().numpy()
    y, s = oracle_gemm_ref(aref, bref, 128, 272, 1024)
    assert (np.abs(out - y) <= gemm_tolerance(y, s, False)).all()
    # and the transform-then-quantize product approximates the plain dY^T X
    plain = to_oracle(dy).astype(np.float64).T @ to_oracle(x).astype(np.float64)
    rel = np.linalg.norm(out - plain) / np.linalg.norm(plain)
    assert rel < 0.2


def test_ldo_larger_than_n():
    x = synth.activation(12, 1, 96, 256)
    w = synth.weight(12, 2, 144, 256)
    aref = oracle.quantize_1d(to_oracle(x), sf_layout=1)
    bref = oracle.quantize_2d(to_oracle(w), sf_layout=1)
    big = torch.full((96, 200), -7.0, device=DEV)
    nv.gemm(upload(aref, 96, 256), upload(bref, 144, 256), out=big[:, :144])
    y, s = oracle_gemm_ref(aref, bref, 96, 144, 256)
    got = big.cpu().numpy()
    assert (np.abs(got[:, :144] - y) <= gemm_tolerance(y, s, False)).all()
    assert (got[:, 144:] == -7.0).all()  # untouched


@pytest.mark.parametrize("T,Nout,Kin", [(200, 320, 256), (130, 3072, 400)])
def test_dgrad_with_transposed_weight_codes(T, Nout, Kin):
    """Data gradient dA = dO . W with W's 2D encoding transposed on the GPU
    (no element re-quantized): the GEMM against the oracle's GEMM on the
    oracle's transposed encoding, fp32 and bf16 outputs."""
    do = synth.activation(13, 1, T, Nout)
    w = synth.weight(13, 2, Nout, Kin)
    qa = nv.quantize_1d(do.to(DEV))
    qwt = nv.transpose_2d(nv.quantize_2d(w.to(DEV)))
    aref = oracle.quantize_1d(to_oracle(do), sf_layout=oracle.SF_TCGEN05)
    wref = oracle.quantize_2d(to_oracle(w), sf_layout=oracle.SF_TCGEN05)
    tc, ts = oracle.transpose_2d(wref[0], wref[1], Nout, Kin, oracle.SF_TCGEN05, oracle.SF_TCGEN05)
    assert_q_equal(qwt, (tc, ts, wref[2]), "W^T")
    y, s = oracle_gemm_ref(aref, (tc, ts, wref[2]), T, Kin, Nout)
    for dt in (torch.float32, torch.bfloat16):
        got = nv.gemm(qa, qwt, out_dtype=dt).float().cpu().numpy().astype(np.float64)
        tol = gemm_tolerance(y, s, dt == torch.bfloat16)
        bad = np.argwhere(np.abs(got - y) > tol)
        assert bad.size == 0, "%d outputs out of tolerance, first %s" % (len(bad), bad[0])


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("epilogue", [nv.NVFP4_EPI_GELU_TANH, nv.NVFP4_EPI_NONE])
def test_output_amax_feeds_the_next_quantization(out_dtype, epilogue):
    """The GEMM records its output's amax (per CTA, in a quantizer workspace);
    quantizing the output from that workspace without an amax pass gives the
    same codes, scales and global scale as the usual two-pass quantization,
    whose global scale is the oracle's; ragged M (300 rows) and N (384)."""
    x = synth.activation(51, 1, 300, 512, device=DEV)
    w = synth.weight(52, 1, 384, 512, device=DEV)
    qa, qb = nv.quantize_1d(x), nv.quantize_2d(w)
    wsq = nv.workspace(1)
    h = nv.gemm(qa, qb, out_dtype=out_dtype, epilogue=epilogue, amax_ws=wsq)
    fused = nv.quantize_1d(h, ws=wsq, amax_ready=True)
    plain = nv.quantize_1d(h)
    torch.cuda.synchronize()
    assert nv.device_error(wsq) == 0
    assert torch.equal(fused.alpha, plain.alpha)
    assert torch.equal(fused.codes, plain.codes)
    assert torch.equal(fused.scales, plain.scales)
    ref_alpha = oracle.quantize_1d(to_oracle(h.cpu()))[2]
    assert float(fused.alpha.cpu()[0]) == np.float32(ref_alpha)



def test_gelu_epilogue_on_exact_products():
    """The epilogue's GELU evaluation alone: with K = 64 and one nonzero
    element per row (E2M1 value times its E4M3 block scale), every output is
    a single product y that the fp32 accumulator holds exactly, swept over
    [-8, 8] (all 16 codes x 8 A scales x 16 B scales).  The fp32 output must
    be within 2^-17 |y| (the evaluation bound stated beside the device code)
    plus its own fp32 rounding of the oracle's double GELU-tanh of y."""
    M, N, K = 128, 256, 64
    kb = K // 16
    a_codes = np.zeros((M, K // 2), np.uint8)
    b_codes = np.zeros((N, K // 2), np.uint8)
    a_codes[:, 0] = np.arange(M) % 16
    b_codes[:, 0] = np.arange(N) % 16
    ea = (0x30 + (np.arange(M) // 16) % 8).astype(np.uint8)   # 0.5 .. 0.9375
    eb = (0x28 + (np.arange(N) // 16) % 16).astype(np.uint8)  # 0.25 .. 0.9375
    a_sf = np.zeros(oracle.sf_bytes(M, kb, oracle.SF_TCGEN05), np.uint8)
    b_sf = np.zeros(oracle.sf_bytes(N, kb, oracle.SF_TCGEN05), np.uint8)
    for r in range(M):
        a_sf[oracle.sf_offset(r, 0, kb, oracle.SF_TCGEN05)] = ea[r]
    for r in range(N):
        b_sf[oracle.sf_offset(r, 0, kb, oracle.SF_TCGEN05)] = eb[r]
    aref, bref = (a_codes, a_sf, 1.0), (b_codes, b_sf, 0.25)
    y, s = oracle_gemm_ref(aref, bref, M, N, K)
    assert np.array_equal(np.abs(y), s) and np.abs(y).max() <= 8.0 and len(np.unique(y)) > 300
    out = nv.gemm(upload(aref, M, K), upload(bref, N, K), out_dtype=torch.float32,
                  epilogue=nv.NVFP4_EPI_GELU_TANH)
    got = out.cpu().numpy().astype(np.float64)
    want = np.vectorize(oracle.gelu_tanh)(y)
    tol = 2.0 ** -17 * np.abs(y) + 2.0 ** -23 * np.abs(want)
    bad = np.argwhere(np.abs(got - want) > tol)
    assert bad.size == 0, "%d outputs, first y=%r gpu=%r ref=%r" % (
        len(bad), y[tuple(bad[0])], got[tuple(bad[0])], want[tuple(bad[0])])


# ------------------------------------------------------------ W4A4 + LoRA
def _lora_inputs(seed, M, N, r):
    u = synth.activation(seed, 101, M, r, n_out=0, std=0.5)     # x A^T, bf16 [M, r]
    bl = synth.weight(seed, 102, N, r)                           # B, bf16 [N, r]
    return u, bl


@pytest.mark.parametrize("M,N,K,r,scale,out_dtype,epi", [
    (64, 128, 256, 128, 1.0, torch.float32, nv.NVFP4_EPI_NONE),      # the tiny linear's shape
    (200, 272, 320, 64, 0.5, torch.bfloat16, nv.NVFP4_EPI_NONE),     # ragged M, N; partial K
    (300, 384, 512, 128, 2.0, torch.bfloat16, nv.NVFP4_EPI_GELU_TANH),
    (257, 512, 3072, 192, -0.75, torch.float32, nv.NVFP4_EPI_NONE),
])
def test_gemm_with_fused_lora_branch(M, N, K, r, scale, out_dtype, epi):
    """out = a b^T (NVFP4) + scale * u bl^T in one GEMM launch against the
    oracle's fp64 GEMM plus its LoRA branch (notes, section 3.4: the quantized
    LoRA linear), |gpu - oracle| <= 1e-3 * (sum |a b| + |scale| sum |u bl|)."""
    x = synth.activation(20, M, M, K)
    w = synth.weight(20, N, N, K)
    aref = oracle.quantize_1d(to_oracle(x), sf_layout=oracle.SF_TCGEN05)
    bref = oracle.quantize_2d(to_oracle(w), sf_layout=oracle.SF_TCGEN05)
    u, bl = _lora_inputs(21, M, N, r)
    ws = nv.workspace(0)
    out = nv.gemm_lora(upload(aref, M, K), upload(bref, N, K), u.to(DEV), bl.to(DEV), scale,
                       out_dtype=out_dtype, epilogue=epi, ws=ws)
    torch.cuda.synchronize()
    assert nv.device_error(ws) == 0
    y, s = oracle_gemm_ref(aref, bref, M, N, K)
    y, s = oracle.lora_add(y, s, to_oracle(u), to_oracle(bl), scale)
    gelu = epi == nv.NVFP4_EPI_GELU_TANH
    if gelu:
        y = np.vectorize(oracle.gelu_tanh)(y)
    got = out.float().cpu().numpy().astype(np.float64)
    tol = gemm_tolerance(y, s, out_dtype == torch.bfloat16, gelu)
    bad = np.argwhere(np.abs(got - y) > tol)
    assert bad.size == 0, "%d outputs out of tolerance, first %s: gpu=%r ref=%r tol=%r" % (
        len(bad), bad[0], got[tuple(bad[0])], y[tuple(bad[0])], tol[tuple(bad[0])])
    # the branch is really there: without it the result is far outside tolerance
    y0, s0 = oracle_gemm_ref(aref, bref, M, N, K)
    if gelu:
        y0 = np.vectorize(oracle.gelu_tanh)(y0)
    assert (np.abs(got - y0) > tol).mean() > 0.5


def test_gemm_lora_qkv_shape_sampled():
    """The DiT QKV projection with a rank-128, scale-1 adapter (the released
    adapter's rank and alpha): the fused GEMM on a sampled grid of outputs."""
    x, w = synth.qkv_linear(DEV)
    M, K = x.shape
    N = w.shape[0]
    ws = nv.workspace(2)
    qa, qb = nv.quantize_mixed([x, w], [False, True], ws=ws)
    u, bl = _lora_inputs(22, M, N, 128)
    out = nv.gemm_lora(qa, qb, u.to(DEV), bl.to(DEV), 1.0, out_dtype=torch.bfloat16, ws=ws)
    torch.cuda.synchronize()
    assert nv.device_error(ws) == 0
    rng = np.random.default_rng(23)
    mi = np.unique(np.concatenate([rng.choice(M, 40, replace=False), [0, M - 1]]))
    ni = np.unique(np.concatenate([rng.choice(N // 16, 3, replace=False) * 16, [0]]))
    ni = (ni[:, None] + np.arange(16)[None, :]).reshape(-1)
    ax, aw = float(qa.alpha.cpu()[0]), float(qb.alpha.cpu()[0])
    xr = oracle.quantize_1d(to_oracle(x.cpu()[torch.from_numpy(mi)]), alpha_in=ax)
    wr = oracle.quantize_2d(to_oracle(w.cpu()[torch.from_numpy(ni)]), alpha_in=aw)
    y, s = oracle.gemm((xr[0], xr[1], ax, oracle.SF_ROWMAJOR), (wr[0], wr[1], aw, oracle.SF_ROWMAJOR),
                       len(mi), len(ni), K)
    y, s = oracle.lora_add(y, s, to_oracle(u)[mi], to_oracle(bl)[ni], 1.0)
    got = out.index_select(0, torch.from_numpy(mi).to(DEV)).index_select(
        1, torch.from_numpy(ni).to(DEV)).float().cpu().numpy().astype(np.float64)
    tol = gemm_tolerance(y, s, True)
    bad = np.argwhere(np.abs(got - y) > tol)
    assert bad.size == 0, "%d of %d out of tolerance" % (len(bad), got.size)


def test_gemm_lora_host_validation():
    """Host-side rules of nvfp4_gemm_lora (nothing is launched)."""
    from nvfp4_block_scaled_20_b200 import capi
    p = 1 << 12
    args = lambda rank, ldu, scale, scr: (p, p, p, p, p, p, 128, 128, 256, p, ldu, p, rank, rank,  # noqa: E731
                                          scale, scr, 1 << 20, p, 0, 128, 0, p, 4096, None)
    assert capi.nvfp4_gemm_lora(*args(96, 96, 1.0, p)) == 2        # rank not a multiple of 64
    assert capi.nvfp4_gemm_lora(*args(128, 100, 1.0, p)) == 2      # ldu < rank... (100 < 128)
    assert capi.nvfp4_gemm_lora(*args(128, 128, float("inf"), p)) == 1
    assert capi.nvfp4_gemm_lora(*args(128, 128, 1.0, p + 8)) == 3  # scratch misaligned
    assert capi.nvfp4_lora_scratch_bytes(2640, 128) == 2640 * 128 * 4


def _split_case(M, N, K, seed):
    x = synth.activation(seed, 1, M, K)
    w = synth.activation(seed, 2, N, K)
    aref = oracle.quantize_1d(to_oracle(x), sf_layout=oracle.SF_TCGEN05)
    bref = oracle.quantize_1d(to_oracle(w), sf_layout=oracle.SF_TCGEN05)
    return aref, bref, upload(aref, M, K), upload(bref, N, K)


@pytest.mark.parametrize("M,N,K", [(256, 512, 8192), (200, 400, 8192)])
def test_split_k_when_tiles_are_fewer_than_pairs(M, N, K):
    """A workspace with partial-sum slabs and fewer tiles than SM pairs: every
    tile is cut along K into ranges of at least eight stages, the ranges'
    fp32 sums added in slab order by the reduction kernel.  Both output types
    within the GEMM bound of the oracle everywhere (ragged M and N included),
    the same bits on a repeat, and the unsplit launch (error-word workspace)
    within the bound too."""
    assert capi.nvfp4_gemm_workspace_bytes(M, N, K, 0) > capi.nvfp4_workspace_bytes(0)
    aref, bref, qa, qb = _split_case(M, N, K, 31)
    y, s = oracle_gemm_ref(aref, bref, M, N, K)
    for dt in (torch.float32, torch.bfloat16):
        ws = nv.gemm_workspace(M, N, K)
        o1 = nv.gemm(qa, qb, out_dtype=dt, ws=ws)
        o2 = nv.gemm(qa, qb, out_dtype=dt, ws=ws)
        plain = nv.gemm(qa, qb, out_dtype=dt, ws=nv.workspace(0))
        torch.cuda.synchronize()
        assert nv.device_error(ws) == 0
        assert torch.equal(o1, o2)
        tol = gemm_tolerance(y, s, dt == torch.bfloat16)
        for got in (o1, plain):
            err = np.abs(got.float().cpu().numpy().astype(np.float64) - y)
            assert (err <= tol).all(), (dt, float((err / np.maximum(tol, 1e-30)).max()))


def test_split_k_of_the_last_partial_round():
    """One tile more than a round of SM pairs (15 x 5 tiles of 256 x 256): the
    first round's tiles run whole and the last one is split along K among the
    idle pairs.  Sampled outputs in every 256 x 256 tile (eight rows and
    eight columns of each tile band, corners included) within the GEMM bound
    of the oracle, whichever tile the schedule left for the last round."""
    M, N, K = 15 * 256, 5 * 256, 8192
    aref, bref, qa, qb = _split_case(M, N, K, 32)
    ws = nv.gemm_workspace(M, N, K)
    out = nv.gemm(qa, qb, out_dtype=torch.float32, ws=ws)
    torch.cuda.synchronize()
    assert nv.device_error(ws) == 0
    rng = np.random.default_rng(5)
    mi = np.unique(np.concatenate([t * 256 + np.r_[0, 255, rng.integers(0, 256, 6)]
                                   for t in range(M // 256)]))
    ni = np.unique(np.concatenate([t * 256 + np.r_[0, 255, rng.integers(0, 256, 6)]
                                   for t in range(N // 256)]))
    gm, gn = np.meshgrid(mi, ni, indexing="ij")
    y, s = oracle_gemm_ref(aref, bref, M, N, K, gm.ravel(), gn.ravel())
    got = out.cpu().numpy()[gm.ravel(), gn.ravel()].astype(np.float64)
    assert (np.abs(got - y) <= gemm_tolerance(y, s, False)).all()
