"""GPU parity at the workloads' full sizes, through the same calls the
benchmark times: DiT QKV projection (2640x9216x3072), the DiT FFN pair
(8192x3072 -> 14336 -> 3072, GELU-tanh between, H's global scale taken from
the up-GEMM's epilogue as the benchmark's step does), the KV cache (60
tensors of 24x32760 tokens x 128, one batched quantize and one batched
dequant; and one layer quantized chunk by chunk, one global scale per chunk
of 8 latent frames), and the weight-gradient path (RHT16 along 32768 tokens,
transposing quantizer, fp32 dW 3072x14336).

Every encoding is checked whole: every global scale exactly (the oracle's
amax over the whole tensor), then every code byte and every scale byte
(tcgen05 padding included) bit-exact against the oracle's encoding of the
same tensor under that global scale.  The oracle is plain single-threaded C;
it runs here on row chunks in a host thread pool (its calls release the
interpreter lock), each chunk a multiple of 128 rows so that the chunk's
scale bytes are one contiguous range in either layout.  The GEMMs are
checked on seeded grids of sampled rows x columns (the fp64 oracle GEMM over
the whole output would take hours) within |gpu - oracle| <= 1e-3 *
sum_k |a_k b_k| (+ half a bf16 ulp for bf16 outputs).  The FFN chain is
checked per stage: its second GEMM's input is the GPU's own GELU output,
re-quantized by the oracle.  Every sample includes the first and last rows,
so the ragged tails are always covered.

Source: the NVFP4 training/inference pages (LongLive-2.0: NVFP4 format,
1D/2D block scaling, 4-over-6 selection, random Hadamard transform on the
weight-gradient path, NVFP4 KV cache with per-chunk global scales)."""
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

try:
    _THREADS = max(1, len(os.sched_getaffinity(0)))
except AttributeError:  # pragma: no cover
    _THREADS = max(1, os.cpu_count() or 1)


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


def host_bits(x: torch.Tensor):
    """The tensor's raw host copy and the exact widening of any slice of it."""
    host = x.detach().cpu()
    if host.dtype == torch.bfloat16:
        return host.view(torch.int16).numpy(), _widen_bf16
    return host.to(torch.float32).numpy(), np.ascontiguousarray


def host_amax(x: torch.Tensor, rht=False, mask=0, block_axis=0, bits=None) -> float:
    """The oracle's amax over a whole device tensor.  A max is order-free, so
    it runs on row chunks (a multiple of 16 rows, keeping the transform's
    groups along rows whole) in the host pool."""
    bits, widen = host_bits(x) if bits is None else bits
    rows = bits.shape[0]
    chunk = max(16, -(-rows // (4 * _THREADS) // 16) * 16)

    def part(r0):
        return oracle.amax(widen(bits[r0:r0 + chunk]), rht=rht, mask=mask, block_axis=block_axis)

    with ThreadPoolExecutor(max_workers=_THREADS) as ex:
        return max(ex.map(part, range(0, rows, chunk)))


def whole_check(q: nv.QTensor, x: torch.Tensor, alpha: float, what: str, two_d=False, rht=False,
                mask=0, block_axis=0, bits=None, dq=None):
    """Every code byte and every scale byte of the GPU encoding q of x against
    the oracle's encoding of x under the global scale alpha, over chunks of
    the encoding's rows (input rows, or input columns for block_axis 1) in
    the host pool.  dq: the GPU's bf16 dequantization of q, checked bit for
    bit against the oracle's dequantization of its own encoding."""
    bits, widen = host_bits(x) if bits is None else bits
    gc = q.codes.cpu().numpy()
    gs = q.scales.cpu().numpy()
    gd = None if dq is None else dq.view(torch.int16).cpu().numpy().view(np.uint16)
    R, kb, layout = q.rows, q.cols // 16, q.sf_layout
    kbg = (kb + 3) // 4
    chunk = max(128, -(-R // (4 * _THREADS) // 128) * 128)

    def sf_range(r0, r1):
        if layout == nv.NVFP4_SF_ROWMAJOR:
            return gs[r0 * kb:r1 * kb]
        start = (r0 // 128) * kbg * 512
        return gs[start:start + -(-(r1 - r0) // 128) * kbg * 512]

    def one(r0):
        r1 = min(R, r0 + chunk)
        src = widen(bits[r0:r1] if block_axis == 0 else bits[:, r0:r1])
        if two_d:
            c, s, _ = oracle.quantize_2d(src, sf_layout=layout, alpha_in=alpha)
        else:
            c, s, _ = oracle.quantize_1d(src, rht=rht, mask=mask, block_axis=block_axis,
                                         sf_layout=layout, alpha_in=alpha)
        msg = (mismatch_report(gc[r0:r1], c, "%s rows %d..%d codes" % (what, r0, r1))
               + mismatch_report(sf_range(r0, r1), s, "%s rows %d..%d scales" % (what, r0, r1)))
        if gd is not None and not msg:
            _, want16 = oracle.dequantize(c, s, alpha, r1 - r0, q.cols, layout)
            msg = mismatch_report(gd[r0:r1], want16, "%s rows %d..%d dequant bits" % (what, r0, r1))
        return msg

    with ThreadPoolExecutor(max_workers=_THREADS) as ex:
        msgs = [m for m in ex.map(one, range(0, R, chunk)) if m]
    assert gc.shape == (R, q.cols // 2)
    assert not msgs, "\n".join(msgs[:4])


def sample_units(n_units: int, k: int, seed: int) -> np.ndarray:
    """k seeded units of range(n_units), always including the first and last."""
    rng = np.random.default_rng(seed)
    pick = rng.choice(n_units, size=min(k, n_units), replace=False)
    return np.unique(np.concatenate([pick, [0, n_units - 1]])).astype(np.int64)


def bands_to_rows(bands: np.ndarray) -> np.ndarray:
    return (bands[:, None] * 16 + np.arange(16)[None, :]).reshape(-1)


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


def rows_of(x: torch.Tensor, idx: np.ndarray) -> np.ndarray:
    return host_f32(x[torch.from_numpy(idx).to(x.device)])


# ------------------------------------------------------------------ QKV
def test_qkv_projection_full():
    """X 2640x3072 (1D) and W 9216x3072 (2D) in the step's mixed call, both
    checked whole; Y on a sampled grid."""
    x, w = synth.qkv_linear(DEV)
    M, K = x.shape
    N = w.shape[0]
    ws = nv.workspace(2)
    qa, qb = nv.quantize_mixed([x, w], [False, True], ws=ws)
    y16 = nv.gemm(qa, qb, out_dtype=torch.bfloat16, ws=ws)
    y32 = nv.gemm(qa, qb, out_dtype=torch.float32, ws=ws)
    torch.cuda.synchronize()
    assert nv.device_error(ws) == 0

    ax = check_alpha(qa, host_amax(x), "X")
    aw = check_alpha(qb, host_amax(w), "W")
    whole_check(qa, x, ax, "X")
    whole_check(qb, w, aw, "W", two_d=True)

    mi = sample_units(M, 48, 21)
    ni = bands_to_rows(sample_units(N // 16, 3, 22))
    xr = oracle.quantize_1d(rows_of(x, mi), alpha_in=ax)
    wr = oracle.quantize_2d(rows_of(w, ni), alpha_in=aw)
    yr, sr = oracle.gemm((xr[0], xr[1], ax, oracle.SF_ROWMAJOR),
                         (wr[0], wr[1], aw, oracle.SF_ROWMAJOR), len(mi), len(ni), K)
    check_gemm(grid(y16, mi, ni), yr, sr, True, what="Y bf16")
    check_gemm(grid(y32, mi, ni), yr, sr, False, what="Y fp32")


# ------------------------------------------------------------------ FFN
def test_ffn_pair_bench_path():
    """The FFN step as the benchmark times it: quantize X, up GEMM + GELU
    recording H's amax in a quantizer workspace, H encoded from that amax
    (no amax pass), down GEMM.  Every encoding whole; the fused H encoding
    also equal to the plain two-pass one; the GEMMs per stage on grids."""
    x, wu, wd = synth.ffn_pair(DEV)
    M, D = x.shape
    Hd = wu.shape[0]
    ws, ws_h = nv.workspace(1), nv.workspace(1)
    qx = nv.quantize_1d(x, ws=ws)
    qu = nv.quantize_2d(wu, ws=ws)
    qd = nv.quantize_2d(wd, ws=ws)
    h = nv.gemm(qx, qu, out_dtype=torch.bfloat16, epilogue=nv.NVFP4_EPI_GELU_TANH, amax_ws=ws_h)
    qh = nv.quantize_1d(h, ws=ws_h, amax_ready=True)
    ws_dn = nv.gemm_workspace(M, D, Hd)  # the down GEMM splits its last round, as benchmarked
    y = nv.gemm(qh, qd, out_dtype=torch.bfloat16, ws=ws_dn)
    qh_plain = nv.quantize_1d(h, ws=ws)
    torch.cuda.synchronize()
    assert nv.device_error(ws) == 0 and nv.device_error(ws_h) == 0 and nv.device_error(ws_dn) == 0
    assert torch.equal(qh.alpha, qh_plain.alpha)
    assert torch.equal(qh.codes, qh_plain.codes)
    assert torch.equal(qh.scales, qh_plain.scales)

    # quantizers: every global scale, every code and scale byte
    ax = check_alpha(qx, host_amax(x), "X")
    au = check_alpha(qu, host_amax(wu), "W_up")
    ad = check_alpha(qd, host_amax(wd), "W_dn")
    whole_check(qx, x, ax, "X")
    whole_check(qu, wu, au, "W_up", two_d=True)
    whole_check(qd, wd, ad, "W_dn", two_d=True)

    # stage (i): up GEMM + GELU-tanh on a sampled grid
    mi = sample_units(M, 62, 31)
    ni = bands_to_rows(sample_units(Hd // 16, 6, 32))
    xr = oracle.quantize_1d(rows_of(x, mi), alpha_in=ax)
    ur = oracle.quantize_2d(rows_of(wu, ni), alpha_in=au)
    yr, sr = oracle.gemm((xr[0], xr[1], ax, oracle.SF_ROWMAJOR),
                         (ur[0], ur[1], au, oracle.SF_ROWMAJOR), len(mi), len(ni), D)
    yr = np.vectorize(oracle.gelu_tanh)(yr)
    check_gemm(grid(h, mi, ni), yr, sr, True, gelu=True, what="H = GELU(X W_up^T)")

    # stage (ii): the oracle re-quantizes the GPU's H, whole
    hb = host_bits(h)
    ah = check_alpha(qh, host_amax(h, bits=hb), "H")
    whole_check(qh, h, ah, "H", bits=hb)

    # stage (iii): down GEMM on those encodings
    nd = bands_to_rows(sample_units(D // 16, 2, 33))
    hr = oracle.quantize_1d(rows_of(h, mi), alpha_in=ah)
    dr = oracle.quantize_2d(rows_of(wd, nd), alpha_in=ad)
    yr, sr = oracle.gemm((hr[0], hr[1], ah, oracle.SF_ROWMAJOR),
                         (dr[0], dr[1], ad, oracle.SF_ROWMAJOR), len(mi), len(nd), Hd)
    check_gemm(grid(y, mi, nd), yr, sr, True, what="Y = H W_dn^T")


# ------------------------------------------------------------------ KV cache
def test_kv_cache_full():
    """All 60 tensors in one batched quantize and one batched dequant; every
    tensor's encoding and bf16 dequantization checked whole."""
    xs = [synth.kv_tensor(3, l, wh, device=DEV) for l in range(30) for wh in range(2)]
    qs = nv.quantize_1d_batched(xs, sf_layout=nv.NVFP4_SF_ROWMAJOR)
    outs = nv.dequantize(qs, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    for i, (x, q, o) in enumerate(zip(xs, qs, outs)):
        hb = host_bits(x)
        a = check_alpha(q, host_amax(x, bits=hb), "KV[%d]" % i)
        whole_check(q, x, a, "KV[%d]" % i, bits=hb, dq=o)
    del xs, qs, outs


def test_kv_cache_chunked_global_scales():
    """The pages' chunkwise KV quantization: one global scale per chunk of
    F_c = 8 latent frames and per layer, the chunk's keys (or values)
    [T_c, H, d] flattened to (T_c * H) x d rows.  One layer's K and V in that
    chunk-major layout (21 frames of 1560 tokens x 24 heads: chunks of 8, 8
    and 5 frames), six chunks in one batched call; each chunk's global scale
    is the oracle's of that chunk alone, and every chunk is checked whole."""
    heads, tokens, frame = 24, 32760, 1560
    bounds = [0, 8 * frame, 16 * frame, tokens]
    xs, chunks = [], []
    for wh in range(2):
        x = synth.kv_tensor(3, 0, wh, device=DEV)  # [heads * tokens, 128], head-major
        x = x.view(heads, tokens, 128).transpose(0, 1).reshape(tokens * heads, 128)  # chunk-major
        xs.append(x)
        chunks += [x[b * heads:e * heads] for b, e in zip(bounds[:-1], bounds[1:])]
    qs = nv.quantize_1d_batched(chunks, sf_layout=nv.NVFP4_SF_ROWMAJOR)
    torch.cuda.synchronize()
    alphas = []
    for i, (c, q) in enumerate(zip(chunks, qs)):
        hb = host_bits(c)
        a = check_alpha(q, host_amax(c, bits=hb), "chunk[%d]" % i)
        alphas.append(a)
        whole_check(q, c, a, "chunk[%d]" % i, bits=hb)
    # the chunks' scales differ (their maxima differ), as the per-chunk form intends
    assert len(set(alphas)) > 1


# ------------------------------------------------------------------ WGRAD
def test_wgrad_full():
    """dW = dY^T X with the transform along tokens on both operands; both
    transposed encodings whole, dW on a sampled grid."""
    dy, x, mask = synth.wgrad(DEV)
    T, Do = dy.shape
    Di = x.shape[1]
    ws = nv.workspace(1)
    qdy = nv.quantize_1d(dy, rht=True, mask=mask, block_axis=1, ws=ws)
    qx = nv.quantize_1d(x, rht=True, mask=mask, block_axis=1, ws=ws)
    # the benchmark's launch: the workspace lets the GEMM split its last round
    ws_g = nv.gemm_workspace(Do, Di, T)
    dw = nv.gemm(qdy, qx, out_dtype=torch.float32, ws=ws_g)
    torch.cuda.synchronize()
    assert nv.device_error(ws) == 0 and nv.device_error(ws_g) == 0
    assert (qdy.rows, qdy.cols, qx.rows, qx.cols) == (Do, T, Di, T)

    db, xb = host_bits(dy), host_bits(x)
    a_dy = check_alpha(qdy, host_amax(dy, rht=True, mask=mask, block_axis=1, bits=db), "dY")
    a_x = check_alpha(qx, host_amax(x, rht=True, mask=mask, block_axis=1, bits=xb), "X")
    whole_check(qdy, dy, a_dy, "dY^T", rht=True, mask=mask, block_axis=1, bits=db)
    whole_check(qx, x, a_x, "X^T", rht=True, mask=mask, block_axis=1, bits=xb)

    mi = sample_units(Do, 22, 51)
    ni = sample_units(Di, 22, 52)
    dyr = oracle.quantize_1d(host_f32(dy[:, torch.from_numpy(mi).to(DEV)]).copy(), rht=True,
                             mask=mask, block_axis=1, alpha_in=a_dy)
    xr = oracle.quantize_1d(host_f32(x[:, torch.from_numpy(ni).to(DEV)]).copy(), rht=True,
                            mask=mask, block_axis=1, alpha_in=a_x)
    yr, sr = oracle.gemm((dyr[0], dyr[1], a_dy, oracle.SF_ROWMAJOR),
                         (xr[0], xr[1], a_x, oracle.SF_ROWMAJOR), len(mi), len(ni), T)
    check_gemm(grid(dw, mi, ni), yr, sr, False, what="dW")


# ------------------------------------------------------------------ DGRAD
def test_dgrad_down_projection_full():
    """dX [8192, 14336] = dY [8192, 3072] . W_dn [3072, 14336] on W_dn's 2D
    encoding transposed on the GPU: the transposed codes and scales whole, dY's
    encoding whole, the GEMM on a sampled grid."""
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
    ad = check_alpha(qd, host_amax(wd), "W_dn")
    whole_check(qd, wd, ad, "W_dn", two_d=True)
    dref = oracle.quantize_2d(host_f32(wd), sf_layout=oracle.SF_TCGEN05, alpha_in=ad)
    tc, ts = oracle.transpose_2d(dref[0], dref[1], D, Hd, oracle.SF_TCGEN05, oracle.SF_TCGEN05)
    msg = (mismatch_report(qt.codes.cpu().numpy(), tc, "W_dn^T codes")
           + mismatch_report(qt.scales.cpu().numpy(), ts, "W_dn^T scales"))
    assert not msg, msg
    ay = check_alpha(qy, host_amax(dy), "dY")
    whole_check(qy, dy, ay, "dY")
    mi = sample_units(dy.shape[0], 62, 61)
    ni = sample_units(Hd, 62, 62)
    yr_enc = oracle.quantize_1d(rows_of(dy, mi), alpha_in=ay)
    sc = np.array([[ts[oracle.sf_offset(int(n), j, D // 16, oracle.SF_TCGEN05)]
                    for j in range(D // 16)] for n in ni], dtype=np.uint8)
    yr, sr = oracle.gemm((yr_enc[0], yr_enc[1], ay, oracle.SF_ROWMAJOR),
                         (tc[ni], sc.reshape(-1), ad, oracle.SF_ROWMAJOR),
                         len(mi), len(ni), D)
    check_gemm(grid(dx, mi, ni), yr, sr, True, what="dX")
