"""GPU parity at the workloads' full sizes, through the same calls the
benchmark times: DiT QKV projection (2640x9216x3072), the DiT FFN pair
(8192x3072 -> 14336 -> 3072, GELU-tanh between), the KV cache (60 tensors of
24x32760 tokens x 128, one batched quantize and one batched dequant), and the
weight-gradient path (RHT16 along 32768 tokens, transposing quantizer, fp32
dW 3072x14336).

The oracle is single-threaded and slow, so beyond the QKV operands (checked
whole) it checks a seeded sample: every global scale exactly (its amax over
the whole tensor), the codes and scale bytes of sampled rows (16-row bands for
2D weights) bit-exact, with the oracle given the global scale it computed
itself, and the GEMM on the grid of sampled rows x sampled columns within
|gpu - oracle| <= 1e-3 * sum_k |a_k b_k| (+ half a bf16 ulp for bf16 outputs).
The FFN chain is checked per stage (its second GEMM's input is the GPU's own
GELU output, re-quantized by the oracle).  Every sample includes the first and
last rows so the ragged tails are always covered.

Source: the NVFP4 training/inference pages (LongLive-2.0: NVFP4 format,
1D/2D block scaling, 4-over-6 selection, random Hadamard transform on the
weight-gradient path, NVFP4 KV cache)."""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
import nvfp4_block_scaled_20_b200 as nv
from nvfp4_block_scaled_20_b200 import synth
from gpu_helpers import DEV, gemm_tolerance, mismatch_report, require_gpu

pytestmark = pytest.mark.gpu

_THREADS = max(1, min(16, os.cpu_count() or 1))


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    yield
    torch.cuda.empty_cache()


def host_f32(t: torch.Tensor) -> np.ndarray:
    """Device tensor -> host, then widened exactly to fp32 on the host."""
    return t.detach().cpu().to(torch.float32).numpy()


def _widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp32 (exact: the 16 bits become the high half)."""
    return (bits.view(np.uint16).astype(np.uint32) << 16).view(np.float32)


def host_amax(x: torch.Tensor, rht=False, mask=0, block_axis=0, chunk_rows=4096) -> float:
    """The oracle's amax over a whole device tensor (a max is order-free, so
    row chunks -- a multiple of 16 rows, keeping the transform's groups along
    rows whole -- run on a few host threads)."""
    host = x.detach().cpu()
    if host.dtype == torch.bfloat16:
        bits = host.view(torch.int16).numpy()
        widen = _widen_bf16
    else:
        bits = host.to(torch.float32).numpy()
        widen = np.ascontiguousarray

    def part(r0):
        return oracle.amax(widen(bits[r0:r0 + chunk_rows]), rht=rht, mask=mask,
                           block_axis=block_axis)

    with ThreadPoolExecutor(max_workers=_THREADS) as ex:
        return max(ex.map(part, range(0, x.shape[0], chunk_rows)))


def sample_units(n_units: int, k: int, seed: int) -> np.ndarray:
    """k seeded units of range(n_units), always including the first and last."""
    rng = np.random.default_rng(seed)
    pick = rng.choice(n_units, size=min(k, n_units), replace=False)
    return np.unique(np.concatenate([pick, [0, n_units - 1]])).astype(np.int64)


def bands_to_rows(bands: np.ndarray) -> np.ndarray:
    return (bands[:, None] * 16 + np.arange(16)[None, :]).reshape(-1)


def gpu_scale_rows(q: nv.QTensor, rows: np.ndarray) -> np.ndarray:
    """The GPU's scale bytes of the given rows as [len(rows), cols/16],
    located through the oracle's own layout function."""
    kb = q.cols // 16
    s = q.scales.cpu().numpy()
    if q.sf_layout == nv.NVFP4_SF_ROWMAJOR:
        return s.reshape(q.rows, kb)[rows]
    off = np.array([[oracle.sf_offset(int(r), j, kb, oracle.SF_TCGEN05) for j in range(kb)]
                    for r in rows], dtype=np.int64)
    return s[off]


def check_rows(q: nv.QTensor, rows: np.ndarray, ref, what: str):
    """Sampled rows of a GPU encoding against the oracle's encoding of the
    same rows (row-major scales)."""
    codes, scales, _ = ref
    kb = q.cols // 16
    gc = q.codes[torch.from_numpy(rows).to(q.codes.device)].cpu().numpy()
    gs = gpu_scale_rows(q, rows)
    msg = (mismatch_report(gc, codes, what + " codes")
           + mismatch_report(gs, scales.reshape(len(rows), kb), what + " scales"))
    assert not msg, msg


def check_alpha(q: nv.QTensor, amax: float, what: str) -> float:
    want = oracle.alpha_from_amax(amax)
    got = float(q.alpha.cpu()[0])
    assert got == np.float32(want), "%s alpha gpu=%r oracle=%r" % (what, got, want)
    return want


def check_gemm(got: np.ndarray, y: np.ndarray, s: np.ndarray, out_bf16: bool, gelu=False,
               what=""):
    tol = gemm_tolerance(y, s, out_bf16, gelu)
    err = np.abs(got.astype(np.float64) - y)
    bad = np.argwhere(err > tol)
    assert bad.size == 0, "%s: %d of %d outputs out of tolerance, first %s gpu=%r ref=%r tol=%r" % (
        what, len(bad), got.size, bad[0], got[tuple(bad[0])], y[tuple(bad[0])],
        tol[tuple(bad[0])])


def grid(out: torch.Tensor, mi: np.ndarray, ni: np.ndarray) -> np.ndarray:
    m = torch.from_numpy(mi).to(out.device)
    n = torch.from_numpy(ni).to(out.device)
    return out.index_select(0, m).index_select(1, n).float().cpu().numpy()


# ------------------------------------------------------------------ QKV
def test_qkv_projection_full():
    """X 2640x3072 (1D) and W 9216x3072 (2D) checked whole; Y sampled."""
    x, w = synth.qkv_linear(DEV)
    M, K = x.shape
    N = w.shape[0]
    ws = nv.workspace(1)
    qa = nv.quantize_1d(x, ws=ws)
    qb = nv.quantize_2d(w, ws=ws)
    y16 = nv.gemm(qa, qb, out_dtype=torch.bfloat16, ws=ws)
    y32 = nv.gemm(qa, qb, out_dtype=torch.float32, ws=ws)
    torch.cuda.synchronize()
    assert nv.device_error(ws) == 0

    aref = oracle.quantize_1d(host_f32(x), sf_layout=oracle.SF_TCGEN05)
    bref = oracle.quantize_2d(host_f32(w), sf_layout=oracle.SF_TCGEN05)
    for q, ref, what in ((qa, aref, "X"), (qb, bref, "W")):
        assert float(q.alpha.cpu()[0]) == np.float32(ref[2]), what
        msg = (mismatch_report(q.codes.cpu().numpy(), ref[0], what + " codes")
               + mismatch_report(q.scales.cpu().numpy(), ref[1], what + " scales"))
        assert not msg, msg

    mi = sample_units(M, 48, 21)
    ni = sample_units(N, 48, 22)
    mm, nn = np.meshgrid(mi, ni, indexing="ij")
    yr, sr = oracle.gemm_pairs((aref[0], aref[1], aref[2], oracle.SF_TCGEN05),
                               (bref[0], bref[1], bref[2], oracle.SF_TCGEN05), K,
                               mm.reshape(-1), nn.reshape(-1))
    yr = yr.reshape(mm.shape)
    sr = sr.reshape(mm.shape)
    check_gemm(grid(y16, mi, ni), yr, sr, True, what="Y bf16")
    check_gemm(grid(y32, mi, ni), yr, sr, False, what="Y fp32")


# ------------------------------------------------------------------ FFN
def test_ffn_pair_per_stage():
    x, wu, wd = synth.ffn_pair(DEV)
    M, D = x.shape
    Hd = wu.shape[0]
    ws = nv.workspace(1)
    qx = nv.quantize_1d(x, ws=ws)
    qu = nv.quantize_2d(wu, ws=ws)
    qd = nv.quantize_2d(wd, ws=ws)
    h = nv.gemm(qx, qu, out_dtype=torch.bfloat16, epilogue=nv.NVFP4_EPI_GELU_TANH, ws=ws)
    qh = nv.quantize_1d(h, ws=ws)
    y = nv.gemm(qh, qd, out_dtype=torch.bfloat16, ws=ws)
    torch.cuda.synchronize()
    assert nv.device_error(ws) == 0

    # quantizers: every global scale; sampled rows / bands bit-exact
    ax = check_alpha(qx, host_amax(x), "X")
    au = check_alpha(qu, host_amax(wu), "W_up")
    ad = check_alpha(qd, host_amax(wd), "W_dn")
    mi = sample_units(M, 62, 31)
    xr = oracle.quantize_1d(host_f32(x[torch.from_numpy(mi).to(DEV)]), alpha_in=ax)
    check_rows(qx, mi, xr, "X")
    ub = sample_units(Hd // 16, 6, 32)
    ur = oracle.quantize_2d(host_f32(wu[torch.from_numpy(bands_to_rows(ub)).to(DEV)]),
                            alpha_in=au)
    check_rows(qu, bands_to_rows(ub), ur, "W_up")
    db = sample_units(D // 16, 2, 33)
    dr = oracle.quantize_2d(host_f32(wd[torch.from_numpy(bands_to_rows(db)).to(DEV)]),
                            alpha_in=ad)
    check_rows(qd, bands_to_rows(db), dr, "W_dn")

    # stage (i): up GEMM + GELU-tanh on the sampled grid
    ni = bands_to_rows(ub)
    yr, sr = oracle.gemm((xr[0], xr[1], ax, oracle.SF_ROWMAJOR),
                         (ur[0], ur[1], au, oracle.SF_ROWMAJOR), len(mi), len(ni), D)
    yr = np.vectorize(oracle.gelu_tanh)(yr)
    check_gemm(grid(h, mi, ni), yr, sr, True, gelu=True, what="H = GELU(X W_up^T)")

    # stage (ii): the oracle re-quantizes the GPU's H
    ah = check_alpha(qh, host_amax(h), "H")
    hr = oracle.quantize_1d(host_f32(h[torch.from_numpy(mi).to(DEV)]), alpha_in=ah)
    check_rows(qh, mi, hr, "H")

    # stage (iii): down GEMM on those encodings
    nd = bands_to_rows(db)
    yr, sr = oracle.gemm((hr[0], hr[1], ah, oracle.SF_ROWMAJOR),
                         (dr[0], dr[1], ad, oracle.SF_ROWMAJOR), len(mi), len(nd), Hd)
    check_gemm(grid(y, mi, nd), yr, sr, True, what="Y = H W_dn^T")


# ------------------------------------------------------------------ KV cache
def test_kv_cache_full():
    """All 60 tensors in one batched quantize and one batched dequant."""
    xs = [synth.kv_tensor(3, l, wh, device=DEV) for l in range(30) for wh in range(2)]
    qs = nv.quantize_1d_batched(xs, sf_layout=nv.NVFP4_SF_ROWMAJOR)
    outs = nv.dequantize(qs, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    rows = xs[0].shape[0]
    for i, (x, q, o) in enumerate(zip(xs, qs, outs)):
        a = check_alpha(q, host_amax(x, chunk_rows=1 << 16), "KV[%d]" % i)
        ri = sample_units(rows, 96, 40 + i)
        idx = torch.from_numpy(ri).to(DEV)
        ref = oracle.quantize_1d(host_f32(x[idx]), alpha_in=a)
        check_rows(q, ri, ref, "KV[%d]" % i)
        _, want16 = oracle.dequantize(ref[0], ref[1], a, len(ri), 128)
        got16 = o[idx].view(torch.int16).cpu().numpy().view(np.uint16)
        msg = mismatch_report(got16, want16, "KV[%d] dequant bf16 bits" % i)
        assert not msg, msg
    del xs, qs, outs


# ------------------------------------------------------------------ WGRAD
def test_wgrad_full():
    """dW = dY^T X with the transform along tokens on both operands."""
    dy, x, mask = synth.wgrad(DEV)
    T, Do = dy.shape
    Di = x.shape[1]
    ws = nv.workspace(1)
    qdy = nv.quantize_1d(dy, rht=True, mask=mask, block_axis=1, ws=ws)
    qx = nv.quantize_1d(x, rht=True, mask=mask, block_axis=1, ws=ws)
    dw = nv.gemm(qdy, qx, out_dtype=torch.float32, ws=ws)
    torch.cuda.synchronize()
    assert nv.device_error(ws) == 0
    assert (qdy.rows, qdy.cols, qx.rows, qx.cols) == (Do, T, Di, T)

    a_dy = check_alpha(qdy, host_amax(dy, rht=True, mask=mask, block_axis=1), "dY")
    a_x = check_alpha(qx, host_amax(x, rht=True, mask=mask, block_axis=1), "X")
    mi = sample_units(Do, 22, 51)
    ni = sample_units(Di, 22, 52)
    dyr = oracle.quantize_1d(host_f32(dy[:, torch.from_numpy(mi).to(DEV)]).copy(), rht=True,
                             mask=mask, block_axis=1, alpha_in=a_dy)
    xr = oracle.quantize_1d(host_f32(x[:, torch.from_numpy(ni).to(DEV)]).copy(), rht=True,
                            mask=mask, block_axis=1, alpha_in=a_x)
    check_rows(qdy, mi, dyr, "dY^T")
    check_rows(qx, ni, xr, "X^T")
    yr, sr = oracle.gemm((dyr[0], dyr[1], a_dy, oracle.SF_ROWMAJOR),
                         (xr[0], xr[1], a_x, oracle.SF_ROWMAJOR), len(mi), len(ni), T)
    check_gemm(grid(dw, mi, ni), yr, sr, False, what="dW")


# ------------------------------------------------------------------ DGRAD
def test_dgrad_down_projection_full():
    """dX [8192, 14336] = dY [8192, 3072] . W_dn [3072, 14336] on W_dn's 2D
    encoding transposed on the GPU: transposed codes and scales whole, the
    GEMM on a sampled grid."""
    _, _, wd = synth.ffn_pair(DEV)
    dy = synth.activation(2, 7, 8192, 3072, n_out=0, std=1e-3, device=DEV)
    ws = nv.workspace(1)
    qd = nv.quantize_2d(wd, ws=ws)
    qt = nv.transpose_2d(qd)
    qy = nv.quantize_1d(dy, ws=ws)
    dx = nv.gemm(qy, qt, out_dtype=torch.bfloat16, ws=ws)
    torch.cuda.synchronize()
    assert nv.device_error(ws) == 0
    D, Hd = wd.shape
    dref = oracle.quantize_2d(host_f32(wd), sf_layout=oracle.SF_TCGEN05)
    tc, ts = oracle.transpose_2d(dref[0], dref[1], D, Hd, oracle.SF_TCGEN05, oracle.SF_TCGEN05)
    msg = (mismatch_report(qt.codes.cpu().numpy(), tc, "W_dn^T codes")
           + mismatch_report(qt.scales.cpu().numpy(), ts, "W_dn^T scales"))
    assert not msg, msg
    ay = check_alpha(qy, host_amax(dy), "dY")
    mi = sample_units(dy.shape[0], 62, 61)
    ni = sample_units(Hd, 62, 62)
    yr_enc = oracle.quantize_1d(host_f32(dy[torch.from_numpy(mi).to(DEV)]), alpha_in=ay)
    check_rows(qy, mi, yr_enc, "dY")
    bt = (tc[ni], None)
    sc = np.array([[ts[oracle.sf_offset(int(n), j, D // 16, oracle.SF_TCGEN05)]
                    for j in range(D // 16)] for n in ni], dtype=np.uint8)
    yr, sr = oracle.gemm((yr_enc[0], yr_enc[1], ay, oracle.SF_ROWMAJOR),
                         (bt[0], sc.reshape(-1), float(qd.alpha.cpu()[0]), oracle.SF_ROWMAJOR),
                         len(mi), len(ni), D)
    check_gemm(grid(dx, mi, ni), yr, sr, True, what="dX")
