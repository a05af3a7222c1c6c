"""C-ABI library: loads, exports every symbol include/nvfp4.h declares, and
the host-side rules (sizes, validation) hold.  No compute call is made: every
call here returns during host-side validation, before any CUDA work."""
import ctypes
import os
import re

import pytest
import torch

from conftest import ROOT
from nvfp4_block_scaled_20_b200 import build, capi


@pytest.fixture(scope="module")
def lib():
    build.build()
    return capi.load()


def declared_symbols():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            src = open(os.path.join(inc, f)).read()
            names |= set(re.findall(r"NVFP4_API\s+[\w\s\*]*?\b(nvfp4_\w+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert names == set(capi.EXPORTED)


def test_size_helpers(lib):
    assert capi.nvfp4_codes_bytes(2640, 3072) == 2640 * 1536
    assert capi.nvfp4_scales_bytes(2640, 3072, capi.NVFP4_SF_ROWMAJOR) == 2640 * 192
    # tcgen05 layout pads rows to 128 and blocks to 4
    assert capi.nvfp4_scales_bytes(2640, 3072, capi.NVFP4_SF_TCGEN05) == 2688 * 192
    assert capi.nvfp4_scales_bytes(64, 80, capi.NVFP4_SF_TCGEN05) == 128 * 8
    assert capi.nvfp4_workspace_bytes(0) >= 4
    assert capi.nvfp4_workspace_bytes(60) >= capi.nvfp4_workspace_bytes(0) + 240
    # the GEMM's split-capable workspace is never below the plain one (the
    # error word, plus one amax slot set with NVFP4_EPI_AMAX); without a
    # device the launch would not split, so it is exactly the plain size
    for M, N, K, epi in [(3072, 14336, 32768, 0), (64, 16, 64, 0), (8192, 14336, 3072, 17)]:
        got = capi.nvfp4_gemm_workspace_bytes(M, N, K, epi)
        plain = capi.nvfp4_workspace_bytes(1 if epi & capi.NVFP4_EPI_AMAX else 0)
        assert got >= plain
        if not torch.cuda.is_available():
            assert got == plain


def test_status_strings(lib):
    assert capi.nvfp4_status_string(0) == "ok"
    for s in range(1, 8):
        assert capi.nvfp4_status_string(s) != "unknown status"


def _qp(**kw):
    d = dict(four_over_six=1, rht_enable=0, rht_sign_mask=0, block_axis=0, sf_layout=1,
             amax_from_workspace=0, global_scale_in=None)
    d.update(kw)
    return capi.nvfp4_qparams(**d)


A = 1 << 20  # a fake, well-aligned address: never dereferenced (validation fails first)


def test_quantize_validation(lib):
    ws = capi.nvfp4_workspace_bytes(1)
    q = capi.nvfp4_quantize_1d
    # NULL input
    assert q(None, 1, 64, 256, 256, _qp(), A, A, A, A, ws, None) == 1
    # cols not a multiple of 16
    assert q(A, 1, 64, 250, 250, _qp(), A, A, A, A, ws, None) == 2
    # misaligned input / leading dimension
    assert q(A + 2, 1, 64, 256, 256, _qp(), A, A, A, A, ws, None) == 3
    assert q(A, 1, 64, 256, 264, _qp(), A, A, A, A, ws, None) == 3
    # transposed path needs rows % 16
    assert q(A, 1, 60, 256, 256, _qp(block_axis=1), A, A, A, A, ws, None) == 2
    # workspace too small
    assert q(A, 1, 64, 256, 256, _qp(), A, A, A, A, 0, None) == 4
    # bad enum values
    assert q(A, 7, 64, 256, 256, _qp(), A, A, A, A, ws, None) == 1
    assert q(A, 1, 64, 256, 256, _qp(sf_layout=3), A, A, A, A, ws, None) == 1
    # 2D: RHT not allowed, rows % 16
    q2 = capi.nvfp4_quantize_2d
    assert q2(A, 1, 64, 256, 256, _qp(rht_enable=1), A, A, A, A, ws, None) == 1
    assert q2(A, 1, 40, 256, 256, _qp(), A, A, A, A, ws, None) == 2


def test_gemm_validation(lib):
    ws = capi.nvfp4_workspace_bytes(0)
    g = capi.nvfp4_gemm
    args = lambda M, N, K, ldo, out_dtype=1, epi=0, wsb=ws, a=A: (
        a, A, A, A, A, A, M, N, K, A, out_dtype, ldo, epi, A, wsb, None)
    assert g(*args(64, 128, 250, 128)) == 2      # K % 64
    assert g(*args(64, 120, 256, 120)) == 2      # N % 16
    assert g(*args(64, 128, 256, 100)) == 2      # ldo < N
    assert g(*args(64, 128, 256, 136, 0)) == 3 or g(*args(64, 128, 256, 132, 1)) == 3
    assert g(*args(64, 128, 256, 128, 5)) == 1   # dtype
    assert g(*args(64, 128, 256, 128, 1, 9)) == 1  # epilogue
    assert g(*args(64, 128, 256, 128, 1, 0, 0)) == 4  # workspace
    assert g(*args(64, 128, 256, 128, 1, 0, ws, A + 8)) == 3  # misaligned codes
    assert g(None, A, A, A, A, A, 64, 128, 256, A, 1, 128, 0, A, ws, None) == 1


def test_batched_and_dequant_validation(lib):
    d = (capi.nvfp4_tensor_desc * 2)()
    d[0] = capi.nvfp4_tensor_desc(A, None, A, A, A, 64, 128, 128)
    d[1] = capi.nvfp4_tensor_desc(A, None, A, A, A, 64, 120, 120)
    ws = capi.nvfp4_workspace_bytes(2)
    assert capi.nvfp4_quantize_1d_batched(d, 2, 1, _qp(), A, ws, None) == 2
    assert capi.nvfp4_quantize_1d_batched(d, 1, 1, _qp(global_scale_in=A), A, ws, None) == 1
    assert capi.nvfp4_quantize_1d_batched(d, 1, 1, _qp(), A, 4, None) == 4
    e = (capi.nvfp4_tensor_desc * 1)()
    e[0] = capi.nvfp4_tensor_desc(None, A, A, A, A, 64, 120, 128)
    assert capi.nvfp4_dequantize(e, 1, 1, 0, None) == 2
    e[0] = capi.nvfp4_tensor_desc(None, None, A, A, A, 64, 128, 128)
    assert capi.nvfp4_dequantize(e, 1, 1, 0, None) == 1


def test_quantize_mixed_validation(lib):
    import ctypes
    d = (capi.nvfp4_tensor_desc * 3)()
    d[0] = capi.nvfp4_tensor_desc(A, None, A, A, A, 64, 128, 128)
    d[1] = capi.nvfp4_tensor_desc(A, None, A, A, A, 40, 128, 128)  # rows % 16 != 0
    d[2] = capi.nvfp4_tensor_desc(A, None, A, A, A, 64, 120, 120)  # cols % 16 != 0
    flags = (ctypes.c_int32 * 3)(0, 1, 0)
    ws = capi.nvfp4_workspace_bytes(3)
    f = capi.nvfp4_quantize_mixed
    # a 40-row tensor is fine in 1D, not in 16x16 tiles
    assert f(d, flags, 2, 1, _qp(), A, ws, None) == 2
    flags[1] = 0
    assert f(d, flags, 3, 1, _qp(), A, ws, None) == 2   # cols % 16
    flags[1] = 2
    assert f(d, flags, 2, 1, _qp(), A, ws, None) == 1   # flag not 0 / 1
    flags[1] = 1
    d[1] = capi.nvfp4_tensor_desc(A, None, A, A, A, 64, 128, 128)
    assert f(d, flags, 2, 1, _qp(rht_enable=1), A, ws, None) == 1
    assert f(d, flags, 2, 1, _qp(block_axis=1), A, ws, None) == 1
    assert f(d, flags, 2, 1, _qp(global_scale_in=A), A, ws, None) == 1
    assert f(d, flags, 2, 1, _qp(), A, capi.nvfp4_workspace_bytes(1), None) == 4
    assert f(d, flags, 65, 1, _qp(), A, capi.nvfp4_workspace_bytes(65), None) == 2
    assert f(d, flags, 0, 1, _qp(), A, ws, None) == 0   # nothing to do
    assert f(None, flags, 2, 1, _qp(), A, ws, None) == 1


def test_output_amax_validation(lib):
    ws0, ws1 = capi.nvfp4_workspace_bytes(0), capi.nvfp4_workspace_bytes(1)
    g = capi.nvfp4_gemm
    args = lambda epi, wsb: (A, A, A, A, A, A, 64, 128, 256, A, 1, 128, epi, A, wsb, None)
    # the output amax needs a quantizer-sized workspace for its partials
    assert g(*args(capi.NVFP4_EPI_AMAX, ws0)) == 4
    assert g(*args(capi.NVFP4_EPI_GELU_TANH | capi.NVFP4_EPI_AMAX, ws0)) == 4
    assert g(*args(2 | capi.NVFP4_EPI_AMAX, ws1)) == 1       # no activation 2
    q = capi.nvfp4_quantize_1d
    assert q(A, 1, 64, 256, 256, _qp(amax_from_workspace=2), A, A, A, A, ws1, None) == 1
    assert q(A, 1, 64, 256, 256, _qp(amax_from_workspace=1, rht_enable=1), A, A, A, A, ws1,
             None) == 1
    # batched, mixed and no-workspace calls take no producer amax
    import ctypes
    d = (capi.nvfp4_tensor_desc * 1)()
    d[0] = capi.nvfp4_tensor_desc(A, None, A, A, A, 64, 128, 128)
    flags = (ctypes.c_int32 * 1)(0)
    assert capi.nvfp4_quantize_1d_batched(d, 1, 1, _qp(amax_from_workspace=1), A, ws1, None) == 1
    assert capi.nvfp4_quantize_mixed(d, flags, 1, 1, _qp(amax_from_workspace=1), A, ws1, None) == 1
    assert capi.nvfp4_quantize_1d_batched_noalloc(d, 1, 1, _qp(amax_from_workspace=1), None) == 1


def test_rht_validation(lib):
    assert capi.nvfp4_rht16(A, 1, 64, 100, 100, 0, 0, A, None) == 2
    assert capi.nvfp4_rht16(A, 1, 60, 64, 64, 1, 0, A, None) == 2
    assert capi.nvfp4_rht16(A, 1, 64, 64, 64, 2, 0, A, None) == 1


def _ranges(pairs):
    flat = [v for p in pairs for v in p]
    return (ctypes.c_int64 * max(1, len(flat)))(*flat)


def test_dequantize_rows_validation(lib):
    e = (capi.nvfp4_tensor_desc * 1)()
    e[0] = capi.nvfp4_tensor_desc(None, A, A, A, A, 64, 128, 128)
    r = _ranges([(0, 8), (32, 40)])
    assert capi.nvfp4_dequantize_rows(e, 1, None, 2, 1, 0, None) == 1   # ranges missing
    assert capi.nvfp4_dequantize_rows(e, 1, _ranges([(-1, 4)]), 1, 1, 0, None) == 2
    assert capi.nvfp4_dequantize_rows(e, 1, _ranges([(9, 4)]), 1, 1, 0, None) == 2
    assert capi.nvfp4_dequantize_rows(e, 1, _ranges([(60, 65)]), 1, 1, 0, None) == 2  # past rows
    assert capi.nvfp4_dequantize_rows(e, 1, r, 1025, 1, 0, None) == 2   # more than 1024 ranges
    assert capi.nvfp4_dequantize_rows(e, 1, r, 2, 7, 0, None) == 1      # unknown dtype
    assert capi.nvfp4_dequantize_rows(e, 1, r, 2, 1, 3, None) == 1      # unknown layout
    e[0] = capi.nvfp4_tensor_desc(None, A, A, A, A, 64, 120, 128)
    assert capi.nvfp4_dequantize_rows(e, 1, r, 2, 1, 0, None) == 2      # cols % 16
    # empty union or no tensors: nothing to do, nothing launched
    assert capi.nvfp4_dequantize_rows(e, 0, r, 2, 1, 0, None) == 0
    e[0] = capi.nvfp4_tensor_desc(None, A, A, A, A, 64, 128, 128)
    assert capi.nvfp4_dequantize_rows(e, 1, _ranges([(5, 5)]), 1, 1, 0, None) == 0


def test_window_rows_helpers_match_a_set_union():
    """The binding's output height and head-wise ranges against a brute-force
    set of row indices."""
    import random
    import nvfp4_block_scaled_20_b200 as nv
    rnd = random.Random(7)
    for _ in range(200):
        rr = []
        for _ in range(rnd.randrange(0, 6)):
            b = rnd.randrange(0, 50)
            rr.append((b, b + rnd.randrange(0, 12)))
        want = set()
        for b, e in rr:
            want.update(range(b, e))
        assert nv.merged_rows(rr) == len(want)
    heads, tokens = 3, 40
    tr = [(0, 4), (10, 14), (30, 40), (12, 20)]
    rows = nv.window_row_ranges(heads, tokens, tr)
    want = {h * tokens + t for h in range(heads) for a, b in tr for t in range(a, b)}
    got = set()
    for b, e in rows:
        got.update(range(b, e))
    assert got == want and nv.merged_rows(rows) == len(want)


def test_transpose_2d_validation(lib):
    assert capi.nvfp4_transpose_2d(A, A, 0, 64, 120, A, A, 0, None) == 2   # cols % 16
    assert capi.nvfp4_transpose_2d(A, A, 0, 60, 128, A, A, 0, None) == 2   # rows % 16
    assert capi.nvfp4_transpose_2d(A, A, 2, 64, 128, A, A, 0, None) == 1   # layout
    assert capi.nvfp4_transpose_2d(None, A, 0, 64, 128, A, A, 0, None) == 1
    assert capi.nvfp4_transpose_2d(A + 4, A, 0, 64, 128, A, A, 0, None) == 3  # codes alignment
    assert capi.nvfp4_transpose_2d(None, None, 0, 0, 128, None, None, 0, None) == 0  # empty
