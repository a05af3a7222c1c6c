"""B200-native NVFP4 W4A4 linear-layer path (sm_100a kernels behind a C ABI).

The compute lives in libnvfp4.so (see include/nvfp4.h).  This package holds
the ctypes binding (``capi``), torch-facing helpers that allocate outputs with
torch and marshal pointers and streams (below), the build step (``build``)
and the seeded input generator (``synth``).  Importing the package does not
load the library; the first call does, and fails loudly if it is missing.
"""
from __future__ import annotations

from dataclasses import dataclass

from . import capi
from .capi import (NVFP4_BF16, NVFP4_EPI_AMAX, NVFP4_EPI_GELU_TANH, NVFP4_EPI_NONE,  # noqa: F401
                   NVFP4_F32,
                   NVFP4_SF_ROWMAJOR, NVFP4_SF_TCGEN05, NVFP4Error)

__all__ = ["QTensor", "quantize_1d", "quantize_2d", "global_scale", "quantize_1d_batched",
           "quantize_mixed", "gemm_lora",
           "dequantize", "dequantize_rows", "window_row_ranges", "transpose_2d", "gemm", "rht16", "workspace",
           "device_error", "capi"]


def _torch():
    import torch
    return torch


def _dtype_code(t):
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return NVFP4_BF16
    if t.dtype == torch.float32:
        return NVFP4_F32
    raise TypeError("unsupported dtype %s" % t.dtype)


def _stream(stream):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


@dataclass
class QTensor:
    """An NVFP4 encoding: packed codes [rows, cols/2] u8, scale bytes in
    ``sf_layout``, and the device fp32 global scale (shape [1])."""
    codes: object
    scales: object
    alpha: object
    rows: int
    cols: int
    sf_layout: int


def workspace(n_tensors: int = 1, device=None):
    torch = _torch()
    return torch.zeros(capi.nvfp4_workspace_bytes(n_tensors), dtype=torch.uint8,
                       device=device or "cuda")


def gemm_workspace(M: int, N: int, K: int, epilogue: int = NVFP4_EPI_NONE, device=None):
    """Workspace for gemm(): nvfp4_gemm_workspace_bytes, error word zeroed (the
    rest needs no initialization).  With it, the tiles of the last partial
    round of the persistent schedule are split along K."""
    torch = _torch()
    ws = torch.empty(capi.nvfp4_gemm_workspace_bytes(M, N, K, epilogue), dtype=torch.uint8,
                     device=device or "cuda")
    ws[:capi.nvfp4_workspace_bytes(0)].zero_()
    return ws


def _qparams(four_over_six, rht, mask, block_axis, sf_layout, alpha_in, amax_ready=False):
    return capi.nvfp4_qparams(int(four_over_six), int(rht), int(mask) & 0xFFFFFFFF,
                              int(block_axis), int(sf_layout), int(bool(amax_ready)),
                              None if alpha_in is None else alpha_in.data_ptr())


def _alloc_q(rows, cols, sf_layout, device):
    torch = _torch()
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=device)
    scales = torch.empty(capi.nvfp4_scales_bytes(rows, cols, sf_layout), dtype=torch.uint8,
                         device=device)
    alpha = torch.empty(1, dtype=torch.float32, device=device)
    return codes, scales, alpha


def quantize_1d(x, four_over_six=True, rht=False, mask=0, block_axis=0,
                sf_layout=NVFP4_SF_TCGEN05, alpha_in=None, ws=None, out=None, stream=None,
                amax_ready=False):
    """nvfp4_quantize_1d on a 2D CUDA tensor (row stride = x.stride(0))."""
    rows, cols = x.shape
    R, C = (rows, cols) if block_axis == 0 else (cols, rows)
    if out is None:
        out = QTensor(*_alloc_q(R, C, sf_layout, x.device), R, C, sf_layout)
    ws = workspace(1, x.device) if ws is None else ws
    qp = _qparams(four_over_six, rht, mask, block_axis, sf_layout, alpha_in, amax_ready)
    st = capi.nvfp4_quantize_1d(x.data_ptr(), _dtype_code(x), rows, cols, x.stride(0), qp,
                                out.codes.data_ptr(), out.scales.data_ptr(), out.alpha.data_ptr(),
                                ws.data_ptr(), ws.numel(), _stream(stream))
    capi.check("nvfp4_quantize_1d", st)
    return out


def quantize_2d(w, four_over_six=True, sf_layout=NVFP4_SF_TCGEN05, alpha_in=None, ws=None,
                out=None, stream=None):
    rows, cols = w.shape
    if out is None:
        out = QTensor(*_alloc_q(rows, cols, sf_layout, w.device), rows, cols, sf_layout)
    ws = workspace(1, w.device) if ws is None else ws
    qp = _qparams(four_over_six, 0, 0, 0, sf_layout, alpha_in)
    st = capi.nvfp4_quantize_2d(w.data_ptr(), _dtype_code(w), rows, cols, w.stride(0), qp,
                                out.codes.data_ptr(), out.scales.data_ptr(), out.alpha.data_ptr(),
                                ws.data_ptr(), ws.numel(), _stream(stream))
    capi.check("nvfp4_quantize_2d", st)
    return out


def global_scale(x, rht=False, mask=0, block_axis=0, ws=None, out=None, stream=None):
    torch = _torch()
    rows, cols = x.shape
    out = torch.empty(1, dtype=torch.float32, device=x.device) if out is None else out
    ws = workspace(1, x.device) if ws is None else ws
    qp = _qparams(1, rht, mask, block_axis, 0, None)
    st = capi.nvfp4_global_scale(x.data_ptr(), _dtype_code(x), rows, cols, x.stride(0), qp,
                                 out.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream))
    capi.check("nvfp4_global_scale", st)
    return out


def quantize_1d_batched(xs, four_over_six=True, sf_layout=NVFP4_SF_ROWMAJOR, ws=None, outs=None,
                        stream=None):
    """One nvfp4_quantize_1d_batched call over a list of 2D tensors."""
    n = len(xs)
    if outs is None:
        outs = [QTensor(*_alloc_q(x.shape[0], x.shape[1], sf_layout, x.device), x.shape[0],
                        x.shape[1], sf_layout) for x in xs]
    ws = workspace(n, xs[0].device) if ws is None else ws
    descs = (capi.nvfp4_tensor_desc * n)()
    for i, (x, q) in enumerate(zip(xs, outs)):
        descs[i] = capi.nvfp4_tensor_desc(x.data_ptr(), None, q.codes.data_ptr(),
                                          q.scales.data_ptr(), q.alpha.data_ptr(), x.shape[0],
                                          x.shape[1], x.stride(0))
    qp = _qparams(four_over_six, 0, 0, 0, sf_layout, None)
    st = capi.nvfp4_quantize_1d_batched(descs, n, _dtype_code(xs[0]), qp, ws.data_ptr(),
                                        ws.numel(), _stream(stream))
    capi.check("nvfp4_quantize_1d_batched", st)
    return outs


def quantize_mixed(xs, two_d, four_over_six=True, sf_layout=NVFP4_SF_TCGEN05, ws=None,
                   outs=None, stream=None):
    """One nvfp4_quantize_mixed call: xs[i] quantized 1D (two_d[i] false) or
    in 16x16 tiles (true), each with the global scale of its own amax."""
    import ctypes
    n = len(xs)
    if outs is None:
        outs = [QTensor(*_alloc_q(x.shape[0], x.shape[1], sf_layout, x.device), x.shape[0],
                        x.shape[1], sf_layout) for x in xs]
    ws = workspace(n, xs[0].device) if ws is None else ws
    descs = (capi.nvfp4_tensor_desc * n)()
    flags = (ctypes.c_int32 * n)()
    for i, (x, q) in enumerate(zip(xs, outs)):
        descs[i] = capi.nvfp4_tensor_desc(x.data_ptr(), None, q.codes.data_ptr(),
                                          q.scales.data_ptr(), q.alpha.data_ptr(), x.shape[0],
                                          x.shape[1], x.stride(0))
        flags[i] = 1 if two_d[i] else 0
    qp = _qparams(four_over_six, 0, 0, 0, sf_layout, None)
    st = capi.nvfp4_quantize_mixed(descs, flags, n, _dtype_code(xs[0]), qp, ws.data_ptr(),
                                   ws.numel(), _stream(stream))
    capi.check("nvfp4_quantize_mixed", st)
    return outs


def dequantize(qs, out_dtype=None, outs=None, stream=None):
    """One nvfp4_dequantize call over a list of QTensor (all of one layout)."""
    torch = _torch()
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    n = len(qs)
    if outs is None:
        outs = [torch.empty((q.rows, q.cols), dtype=out_dtype, device=q.codes.device) for q in qs]
    descs = (capi.nvfp4_tensor_desc * n)()
    for i, (q, o) in enumerate(zip(qs, outs)):
        descs[i] = capi.nvfp4_tensor_desc(None, o.data_ptr(), q.codes.data_ptr(),
                                          q.scales.data_ptr(), q.alpha.data_ptr(), q.rows, q.cols,
                                          o.stride(0))
    code = NVFP4_BF16 if out_dtype == torch.bfloat16 else NVFP4_F32
    st = capi.nvfp4_dequantize(descs, n, code, qs[0].sf_layout, _stream(stream))
    capi.check("nvfp4_dequantize", st)
    return outs


def merged_rows(row_ranges):
    """Number of rows in the union of half-open ranges (the output height of
    dequantize_rows)."""
    total, end = 0, None
    for b, e in sorted((int(b), int(e)) for b, e in row_ranges if int(e) > int(b)):
        if end is None or b > end:
            total += e - b
            end = e
        elif e > end:
            total += e - end
            end = e
    return total


def window_row_ranges(heads, tokens, token_ranges):
    """Row ranges of a [heads * tokens, d] cache for the given token ranges of
    every head (e.g. global sink, shot sink, recent window)."""
    return [(h * tokens + a, h * tokens + b) for h in range(heads) for a, b in token_ranges]


def dequantize_rows(qs, row_ranges, out_dtype=None, outs=None, stream=None):
    """One nvfp4_dequantize_rows call: the union of row_ranges of every
    QTensor, in row order, into contiguous outputs."""
    import ctypes
    torch = _torch()
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    n = len(qs)
    rows_out = merged_rows(row_ranges)
    if outs is None:
        outs = [torch.empty((rows_out, q.cols), dtype=out_dtype, device=q.codes.device) for q in qs]
    descs = (capi.nvfp4_tensor_desc * n)()
    for i, (q, o) in enumerate(zip(qs, outs)):
        descs[i] = capi.nvfp4_tensor_desc(None, o.data_ptr(), q.codes.data_ptr(),
                                          q.scales.data_ptr(), q.alpha.data_ptr(), q.rows, q.cols,
                                          o.stride(0))
    flat = (ctypes.c_int64 * (2 * len(row_ranges)))(*[v for r in row_ranges for v in r])
    code = NVFP4_BF16 if out_dtype == torch.bfloat16 else NVFP4_F32
    st = capi.nvfp4_dequantize_rows(descs, n, flat, len(row_ranges), code, qs[0].sf_layout,
                                    _stream(stream))
    capi.check("nvfp4_dequantize_rows", st)
    return outs


def transpose_2d(q: QTensor, sf_layout=None, out=None, stream=None):
    """The encoding of the transpose of a 2D-quantized matrix (codes
    transposed, tile scales carried over, global scale shared)."""
    sf_layout = q.sf_layout if sf_layout is None else sf_layout
    if out is None:
        codes, scales, _ = _alloc_q(q.cols, q.rows, sf_layout, q.codes.device)
        out = QTensor(codes, scales, q.alpha, q.cols, q.rows, sf_layout)
    st = capi.nvfp4_transpose_2d(q.codes.data_ptr(), q.scales.data_ptr(), q.sf_layout, q.rows,
                                 q.cols, out.codes.data_ptr(), out.scales.data_ptr(), sf_layout,
                                 _stream(stream))
    capi.check("nvfp4_transpose_2d", st)
    return out


def gemm(a: QTensor, b: QTensor, out_dtype=None, epilogue=NVFP4_EPI_NONE, out=None, ws=None,
         stream=None, amax_ws=None):
    """out[M, N] = a (M x K) times b (N x K) transposed, both NVFP4 (tcgen05 layout).
    amax_ws: a quantizer workspace (workspace(1)) that receives the output's
    amax, for quantize_1d(out, ws=amax_ws, amax_ready=True); it is then the
    GEMM's workspace too (ws must be None or the same tensor)."""
    torch = _torch()
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    M, K = a.rows, a.cols
    N = b.rows
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=a.codes.device)
    if amax_ws is not None:
        if ws is not None and ws is not amax_ws:
            raise ValueError("with amax_ws the GEMM uses that workspace")
        ws, epilogue = amax_ws, epilogue | NVFP4_EPI_AMAX
    ws = gemm_workspace(M, N, K, epilogue, a.codes.device) if ws is None else ws
    code = NVFP4_BF16 if out.dtype == torch.bfloat16 else NVFP4_F32
    st = capi.nvfp4_gemm(a.codes.data_ptr(), a.scales.data_ptr(), a.alpha.data_ptr(),
                         b.codes.data_ptr(), b.scales.data_ptr(), b.alpha.data_ptr(), M, N, K,
                         out.data_ptr(), code, out.stride(0), epilogue, ws.data_ptr(), ws.numel(),
                         _stream(stream))
    capi.check("nvfp4_gemm", st)
    return out


def gemm_lora(a: QTensor, b: QTensor, lora_u, lora_b, lora_scale, out_dtype=None,
              epilogue=NVFP4_EPI_NONE, out=None, ws=None, scratch=None, stream=None):
    """nvfp4_gemm_lora: out = a b^T (NVFP4) + lora_scale * lora_u lora_b^T, the
    adapter branch (bf16 lora_u [M, r] = x A^T, lora_b [N, r]) fused into the
    same GEMM."""
    torch = _torch()
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    M, K = a.rows, a.cols
    N = b.rows
    rank = lora_u.shape[1]
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=a.codes.device)
    ws = workspace(0, a.codes.device) if ws is None else ws
    if scratch is None:
        scratch = torch.empty(capi.nvfp4_lora_scratch_bytes(M, rank), dtype=torch.uint8,
                              device=a.codes.device)
    code = NVFP4_BF16 if out.dtype == torch.bfloat16 else NVFP4_F32
    st = capi.nvfp4_gemm_lora(a.codes.data_ptr(), a.scales.data_ptr(), a.alpha.data_ptr(),
                              b.codes.data_ptr(), b.scales.data_ptr(), b.alpha.data_ptr(), M, N, K,
                              lora_u.data_ptr(), lora_u.stride(0), lora_b.data_ptr(),
                              lora_b.stride(0), rank, float(lora_scale), scratch.data_ptr(),
                              scratch.numel(), out.data_ptr(), code, out.stride(0), epilogue,
                              ws.data_ptr(), ws.numel(), _stream(stream))
    capi.check("nvfp4_gemm_lora", st)
    return out


def rht16(x, block_axis=0, mask=0, out=None, stream=None):
    torch = _torch()
    rows, cols = x.shape
    out = torch.empty((rows, cols), dtype=torch.float32, device=x.device) if out is None else out
    st = capi.nvfp4_rht16(x.data_ptr(), _dtype_code(x), rows, cols, x.stride(0), block_axis, mask,
                          out.data_ptr(), _stream(stream))
    capi.check("nvfp4_rht16", st)
    return out


def device_error(ws, stream=None) -> int:
    st, v = capi.nvfp4_get_device_error(ws.data_ptr(), _stream(stream))
    capi.check("nvfp4_get_device_error", st)
    return v
