"""ctypes declarations of the C ABI in include/nvfp4.h (libnvfp4.so).

Each function here has the C name and the C argument list (pointers as Python
ints, streams as ints); nothing is computed in Python.  Loading fails loudly
when the library is missing: there is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnvfp4.so")

NVFP4_OK = 0
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "SHAPE", 3: "ALIGN", 4: "WORKSPACE", 5: "CUDA",
                6: "TIMEOUT", 7: "UNSUPPORTED"}
NVFP4_F32, NVFP4_BF16 = 0, 1
NVFP4_SF_ROWMAJOR, NVFP4_SF_TCGEN05 = 0, 1
NVFP4_EPI_NONE, NVFP4_EPI_GELU_TANH, NVFP4_EPI_AMAX = 0, 1, 16

EXPORTED = [
    "nvfp4_workspace_bytes", "nvfp4_codes_bytes", "nvfp4_scales_bytes", "nvfp4_global_scale",
    "nvfp4_quantize_1d", "nvfp4_quantize_2d", "nvfp4_quantize_1d_batched", "nvfp4_quantize_mixed",
    "nvfp4_quantize_1d_batched_noalloc", "nvfp4_dequantize", "nvfp4_dequantize_rows",
    "nvfp4_transpose_2d",
    "nvfp4_gemm", "nvfp4_rht16", "nvfp4_get_device_error", "nvfp4_status_string",
    "nvfp4_convert_sweep", "nvfp4_set_wait_limit", "nvfp4_set_test_stall",
    "nvfp4_lora_scratch_bytes", "nvfp4_gemm_lora", "nvfp4_gemm_workspace_bytes",
]


class nvfp4_qparams(ctypes.Structure):
    _fields_ = [("four_over_six", ctypes.c_int32), ("rht_enable", ctypes.c_int32),
                ("rht_sign_mask", ctypes.c_uint32), ("block_axis", ctypes.c_int32),
                ("sf_layout", ctypes.c_int32), ("amax_from_workspace", ctypes.c_int32),
                ("global_scale_in", ctypes.c_void_p)]


class nvfp4_tensor_desc(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("out", ctypes.c_void_p), ("codes", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("global_scale", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("ld", ctypes.c_int64)]


class NVFP4Error(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__("%s failed: %s (%d)" % (fn, STATUS_NAMES.get(status, "?"), status))


_lib = None
_V, _I32, _I64, _U32, _SZ = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32,
                             ctypes.c_size_t)
_QP = ctypes.POINTER(nvfp4_qparams)
_TD = ctypes.POINTER(nvfp4_tensor_desc)

_SIGS = {
    "nvfp4_workspace_bytes": (_SZ, [_I32]),
    "nvfp4_codes_bytes": (_I64, [_I64, _I64]),
    "nvfp4_scales_bytes": (_I64, [_I64, _I64, _I32]),
    "nvfp4_global_scale": (_I32, [_V, _I32, _I64, _I64, _I64, _QP, _V, _V, _SZ, _V]),
    "nvfp4_quantize_1d": (_I32, [_V, _I32, _I64, _I64, _I64, _QP, _V, _V, _V, _V, _SZ, _V]),
    "nvfp4_quantize_2d": (_I32, [_V, _I32, _I64, _I64, _I64, _QP, _V, _V, _V, _V, _SZ, _V]),
    "nvfp4_quantize_1d_batched": (_I32, [_TD, _I32, _I32, _QP, _V, _SZ, _V]),
    "nvfp4_quantize_mixed": (_I32, [_TD, ctypes.POINTER(ctypes.c_int32), _I32, _I32, _QP, _V, _SZ,
                                    _V]),
    "nvfp4_quantize_1d_batched_noalloc": (_I32, [_TD, _I32, _I32, _QP, _V]),
    "nvfp4_dequantize": (_I32, [_TD, _I32, _I32, _I32, _V]),
    "nvfp4_transpose_2d": (_I32, [_V, _V, _I32, _I64, _I64, _V, _V, _I32, _V]),
    "nvfp4_dequantize_rows": (_I32, [_TD, _I32, ctypes.POINTER(ctypes.c_int64), _I32, _I32, _I32,
                                     _V]),
    "nvfp4_gemm": (_I32, [_V, _V, _V, _V, _V, _V, _I64, _I64, _I64, _V, _I32, _I64, _I32, _V,
                          _SZ, _V]),
    "nvfp4_rht16": (_I32, [_V, _I32, _I64, _I64, _I64, _I32, _U32, _V, _V]),
    "nvfp4_get_device_error": (_I32, [_V, ctypes.POINTER(ctypes.c_int32), _V]),
    "nvfp4_status_string": (ctypes.c_char_p, [_I32]),
    "nvfp4_convert_sweep": (_I32, [_I32, _U32, _I64, _V, _V]),
    "nvfp4_set_wait_limit": (_I32, [ctypes.c_uint64]),
    "nvfp4_set_test_stall": (_I32, [_I32]),
    "nvfp4_lora_scratch_bytes": (_SZ, [_I64, _I64]),
    "nvfp4_gemm_workspace_bytes": (_SZ, [_I64, _I64, _I64, _I32]),
    "nvfp4_gemm_lora": (_I32, [_V, _V, _V, _V, _V, _V, _I64, _I64, _I64, _V, _I64, _V, _I64, _I64,
                               ctypes.c_float, _V, _SZ, _V, _I32, _I64, _I32, _V, _SZ, _V]),
}


def load(path: str = LIB_PATH):
    """Load libnvfp4.so (raises OSError if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise OSError("libnvfp4.so not built (%s); run python -m "
                          "nvfp4_block_scaled_20_b200.build" % path)
        L = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def check(fn: str, status: int) -> None:
    if status != NVFP4_OK:
        raise NVFP4Error(fn, status)


def _call(name, *args):
    return getattr(load(), name)(*args)


def nvfp4_workspace_bytes(n):
    return _call("nvfp4_workspace_bytes", n)


def nvfp4_codes_bytes(rows, cols):
    return _call("nvfp4_codes_bytes", rows, cols)


def nvfp4_scales_bytes(rows, cols, layout):
    return _call("nvfp4_scales_bytes", rows, cols, layout)


def nvfp4_global_scale(x, dtype, rows, cols, ld, qp, gs_out, ws, ws_bytes, stream):
    return _call("nvfp4_global_scale", x, dtype, rows, cols, ld, ctypes.byref(qp), gs_out, ws,
                 ws_bytes, stream)


def nvfp4_quantize_1d(x, dtype, rows, cols, ld, qp, codes, scales, gs_out, ws, ws_bytes, stream):
    return _call("nvfp4_quantize_1d", x, dtype, rows, cols, ld, ctypes.byref(qp), codes, scales,
                 gs_out, ws, ws_bytes, stream)


def nvfp4_quantize_2d(x, dtype, rows, cols, ld, qp, codes, scales, gs_out, ws, ws_bytes, stream):
    return _call("nvfp4_quantize_2d", x, dtype, rows, cols, ld, ctypes.byref(qp), codes, scales,
                 gs_out, ws, ws_bytes, stream)


def nvfp4_quantize_1d_batched(descs, n, dtype, qp, ws, ws_bytes, stream):
    return _call("nvfp4_quantize_1d_batched", descs, n, dtype, ctypes.byref(qp), ws, ws_bytes,
                 stream)


def nvfp4_quantize_mixed(descs, two_d, n, dtype, qp, ws, ws_bytes, stream):
    return _call("nvfp4_quantize_mixed", descs, two_d, n, dtype, ctypes.byref(qp), ws, ws_bytes,
                 stream)


def nvfp4_quantize_1d_batched_noalloc(descs, n, dtype, qp, stream):
    """Batched quantization with the library's own fixed scratch (no workspace)."""
    return _call("nvfp4_quantize_1d_batched_noalloc", descs, n, dtype, ctypes.byref(qp), stream)


def nvfp4_dequantize(descs, n, out_dtype, sf_layout, stream):
    return _call("nvfp4_dequantize", descs, n, out_dtype, sf_layout, stream)


def nvfp4_transpose_2d(codes, scales, sf_layout_in, rows, cols, out_codes, out_scales,
                       sf_layout_out, stream):
    return _call("nvfp4_transpose_2d", codes, scales, sf_layout_in, rows, cols, out_codes,
                 out_scales, sf_layout_out, stream)


def nvfp4_dequantize_rows(descs, n, row_ranges, n_ranges, out_dtype, sf_layout, stream):
    return _call("nvfp4_dequantize_rows", descs, n, row_ranges, n_ranges, out_dtype, sf_layout,
                 stream)


def nvfp4_gemm(a_codes, a_sf, a_alpha, b_codes, b_sf, b_alpha, M, N, K, out, out_dtype, ldo,
               epilogue, ws, ws_bytes, stream):
    return _call("nvfp4_gemm", a_codes, a_sf, a_alpha, b_codes, b_sf, b_alpha, M, N, K, out,
                 out_dtype, ldo, epilogue, ws, ws_bytes, stream)


def nvfp4_gemm_workspace_bytes(M, N, K, epilogue):
    return _call("nvfp4_gemm_workspace_bytes", M, N, K, epilogue)


def nvfp4_lora_scratch_bytes(M, rank):
    return _call("nvfp4_lora_scratch_bytes", M, rank)


def nvfp4_gemm_lora(a_codes, a_sf, a_alpha, b_codes, b_sf, b_alpha, M, N, K, lora_u, ldu, lora_b,
                    ldl, rank, lora_scale, scratch, scratch_bytes, out, out_dtype, ldo, epilogue,
                    ws, ws_bytes, stream):
    return _call("nvfp4_gemm_lora", a_codes, a_sf, a_alpha, b_codes, b_sf, b_alpha, M, N, K,
                 lora_u, ldu, lora_b, ldl, rank, lora_scale, scratch, scratch_bytes, out,
                 out_dtype, ldo, epilogue, ws, ws_bytes, stream)


def nvfp4_rht16(x, dtype, rows, cols, ld, block_axis, mask, out, stream):
    return _call("nvfp4_rht16", x, dtype, rows, cols, ld, block_axis, mask, out, stream)


def nvfp4_get_device_error(ws, stream):
    v = ctypes.c_int32(0)
    st = _call("nvfp4_get_device_error", ws, ctypes.byref(v), stream)
    return st, v.value


def nvfp4_convert_sweep(target, first_bits, count, out, stream):
    return _call("nvfp4_convert_sweep", target, first_bits, count, out, stream)


def nvfp4_set_wait_limit(ns):
    return _call("nvfp4_set_wait_limit", ns)


def nvfp4_set_test_stall(on):
    return _call("nvfp4_set_test_stall", on)


def nvfp4_status_string(s):
    return _call("nvfp4_status_string", s).decode()
