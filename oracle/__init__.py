"""CPU oracle for the NVFP4 W4A4 linear path -- test infrastructure.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline
(and ``--impl reference``) leg may import this package.  It wraps the plain C
implementation in ``nvfp4_oracle.c`` (built with gcc, ``-ffp-contract=off``),
which shares nothing with the CUDA library.  Every function takes and
returns numpy arrays; bf16 inputs are passed widened to float32 (exact).

All arithmetic lives in the C file; this module only marshals arguments.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

SF_ROWMAJOR = 0
SF_TCGEN05 = 1

_F32P = ctypes.POINTER(ctypes.c_float)
_U8P = ctypes.POINTER(ctypes.c_uint8)
_U16P = ctypes.POINTER(ctypes.c_uint16)
_F64P = ctypes.POINTER(ctypes.c_double)
_I64P = ctypes.POINTER(ctypes.c_int64)
_i64 = ctypes.c_int64
_i32 = ctypes.c_int
_u32 = ctypes.c_uint32


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to the source (gcc, -O2, no FP contraction)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
           "-fno-builtin", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        L.orc_e2m1_value.restype = ctypes.c_double
        L.orc_e2m1_value.argtypes = [_i32]
        L.orc_e2m1_encode.restype = _i32
        L.orc_e2m1_encode.argtypes = [ctypes.c_float]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_decode.argtypes = [_i32]
        L.orc_e4m3_encode.restype = _i32
        L.orc_e4m3_encode.argtypes = [ctypes.c_float]
        L.orc_e2m1_encode_bits.restype = None
        L.orc_e2m1_encode_bits.argtypes = [_u32, _i64, _U8P]
        L.orc_e4m3_encode_bits.restype = None
        L.orc_e4m3_encode_bits.argtypes = [_u32, _i64, _U8P]
        L.orc_bf16_rne.restype = ctypes.c_uint16
        L.orc_bf16_rne.argtypes = [ctypes.c_float]
        L.orc_rht16_block.restype = None
        L.orc_rht16_block.argtypes = [_F32P, _u32]
        L.orc_rht16.restype = _i32
        L.orc_rht16.argtypes = [_F32P, _i64, _i64, _i64, _i32, _u32, _F32P]
        L.orc_alpha_from_amax.restype = ctypes.c_float
        L.orc_alpha_from_amax.argtypes = [ctypes.c_float]
        L.orc_sf_offset.restype = _i64
        L.orc_sf_offset.argtypes = [_i64, _i64, _i64, _i32]
        L.orc_sf_bytes.restype = _i64
        L.orc_sf_bytes.argtypes = [_i64, _i64, _i32]
        L.orc_amax.restype = ctypes.c_float
        L.orc_amax.argtypes = [_F32P, _i64, _i64, _i64, _i32, _u32, _i32]
        L.orc_quantize_1d.restype = _i32
        L.orc_quantize_1d.argtypes = [_F32P, _i64, _i64, _i64, _i32, _i32, _u32, _i32,
                                      _i32, _F32P, _U8P, _U8P, _F32P]
        L.orc_quantize_2d.restype = _i32
        L.orc_quantize_2d.argtypes = [_F32P, _i64, _i64, _i64, _i32, _i32, _F32P,
                                      _U8P, _U8P, _F32P]
        L.orc_dequantize.restype = None
        L.orc_dequantize.argtypes = [_U8P, _U8P, ctypes.c_float, _i64, _i64, _i32,
                                     _F32P, _U16P]
        L.orc_gemm_pairs.restype = None
        L.orc_gemm_pairs.argtypes = [_U8P, _U8P, ctypes.c_float, _i32, _U8P, _U8P,
                                     ctypes.c_float, _i32, _i64, _i64, _I64P, _I64P,
                                     _F64P, _F64P]
        L.orc_gemm.restype = None
        L.orc_gemm.argtypes = [_U8P, _U8P, ctypes.c_float, _i32, _U8P, _U8P,
                               ctypes.c_float, _i32, _i64, _i64, _i64, _F64P, _F64P]
        L.orc_lora_add.restype = None
        L.orc_lora_add.argtypes = [_F32P, _F32P, _i64, _i64, _i64, ctypes.c_double, _F64P, _F64P]
        L.orc_gelu_tanh.restype = ctypes.c_double
        L.orc_gelu_tanh.argtypes = [ctypes.c_double]
        L.orc_transpose_2d.restype = _i32
        L.orc_transpose_2d.argtypes = [_U8P, _U8P, _i64, _i64, _i32, _U8P, _U8P, _i32]
        _lib = L
    return _lib


def _p(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def _f32(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float32)


# ---------------------------------------------------------------- codecs
def e2m1_value(code: int) -> float:
    return lib().orc_e2m1_value(int(code))


def e2m1_encode(v: float) -> int:
    return lib().orc_e2m1_encode(float(v))


def e4m3_decode(code: int) -> float:
    return lib().orc_e4m3_decode(int(code))


def e4m3_encode(t: float) -> int:
    return lib().orc_e4m3_encode(float(t))


def encode_bits(target: int, first_bits: int, n: int) -> np.ndarray:
    """The oracle's cast of every fp32 with bit pattern first_bits + i,
    i < n: target 0 the E2M1 code, 1 the E4M3 code (uint8 each)."""
    out = np.empty(n, dtype=np.uint8)
    f = lib().orc_e2m1_encode_bits if target == 0 else lib().orc_e4m3_encode_bits
    f(first_bits, n, _p(out, _U8P))
    return out


def bf16_rne(f: float) -> int:
    return lib().orc_bf16_rne(float(f))


def alpha_from_amax(amax: float) -> float:
    return lib().orc_alpha_from_amax(float(amax))


def sf_offset(r: int, kb: int, kb_total: int, layout: int) -> int:
    return lib().orc_sf_offset(r, kb, kb_total, layout)


def sf_bytes(rows: int, kb_total: int, layout: int) -> int:
    return lib().orc_sf_bytes(rows, kb_total, layout)


def lora_add(y, s, u, bl, scale: float):
    """W4A4 + LoRA: (y + scale * u bl^T, s + |scale| * sum |u bl|) for a base
    GEMM's (y, s) [M, N], u = x A^T [M, r] and bl = B [N, r] (fp32 / widened
    bf16).  Returns new arrays; the inputs are not modified."""
    y = np.array(y, dtype=np.float64, copy=True, order="C")
    s = np.array(s, dtype=np.float64, copy=True, order="C")
    u = np.ascontiguousarray(u, dtype=np.float32)
    bl = np.ascontiguousarray(bl, dtype=np.float32)
    M, r = u.shape
    N = bl.shape[0]
    if bl.shape[1] != r or y.shape != (M, N) or s.shape != (M, N):
        raise ValueError("shapes: y, s [M, N], u [M, r], bl [N, r]")
    lib().orc_lora_add(_p(u, _F32P), _p(bl, _F32P), M, N, r, float(scale), _p(y, _F64P),
                       _p(s, _F64P))
    return y, s


def gelu_tanh(x: float) -> float:
    return lib().orc_gelu_tanh(float(x))


# ---------------------------------------------------------------- RHT
def rht16_block(v, mask: int) -> np.ndarray:
    a = _f32(v).copy()
    assert a.size == 16
    lib().orc_rht16_block(_p(a, _F32P), mask)
    return a


def rht16(x, block_axis: int, mask: int) -> np.ndarray:
    x = _f32(x)
    rows, cols = x.shape
    out = np.empty_like(x)
    rc = lib().orc_rht16(_p(x, _F32P), rows, cols, cols, block_axis, mask, _p(out, _F32P))
    if rc != 0:
        raise ValueError("bad shape for rht16")
    return out


def amax(x, rht: bool = False, mask: int = 0, block_axis: int = 0) -> float:
    x = _f32(x)
    rows, cols = x.shape
    return lib().orc_amax(_p(x, _F32P), rows, cols, cols, int(rht), mask, block_axis)


# ---------------------------------------------------------------- quantize
def quantize_1d(x, four_over_six: bool = True, rht: bool = False, mask: int = 0,
                block_axis: int = 0, sf_layout: int = SF_ROWMAJOR, alpha_in=None):
    """Returns (codes [R, C/2] u8, scales (flat, sf layout) u8, alpha float).

    block_axis 0: R, C = rows, cols.  block_axis 1: R, C = cols, rows.
    """
    x = _f32(x)
    rows, cols = x.shape
    R, C = (rows, cols) if block_axis == 0 else (cols, rows)
    codes = np.zeros((R, C // 2), dtype=np.uint8)
    scales = np.zeros(sf_bytes(R, C // 16, sf_layout), dtype=np.uint8)
    a_out = np.zeros(1, dtype=np.float32)
    a_in = None if alpha_in is None else np.array([alpha_in], dtype=np.float32)
    rc = lib().orc_quantize_1d(_p(x, _F32P), rows, cols, cols, int(four_over_six),
                               int(rht), mask, block_axis, sf_layout,
                               None if a_in is None else _p(a_in, _F32P),
                               _p(codes, _U8P), _p(scales, _U8P), _p(a_out, _F32P))
    if rc != 0:
        raise ValueError("bad shape for quantize_1d")
    return codes, scales, float(a_out[0])


def quantize_2d(x, four_over_six: bool = True, sf_layout: int = SF_ROWMAJOR,
                alpha_in=None):
    x = _f32(x)
    rows, cols = x.shape
    codes = np.zeros((rows, cols // 2), dtype=np.uint8)
    scales = np.zeros(sf_bytes(rows, cols // 16, sf_layout), dtype=np.uint8)
    a_out = np.zeros(1, dtype=np.float32)
    a_in = None if alpha_in is None else np.array([alpha_in], dtype=np.float32)
    rc = lib().orc_quantize_2d(_p(x, _F32P), rows, cols, cols, int(four_over_six),
                               sf_layout, None if a_in is None else _p(a_in, _F32P),
                               _p(codes, _U8P), _p(scales, _U8P), _p(a_out, _F32P))
    if rc != 0:
        raise ValueError("bad shape for quantize_2d")
    return codes, scales, float(a_out[0])


def dequantize(codes, scales, alpha: float, rows: int, cols: int,
               sf_layout: int = SF_ROWMAJOR):
    """Returns (fp32 [rows, cols], bf16 bits [rows, cols] as uint16)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    out32 = np.empty((rows, cols), dtype=np.float32)
    out16 = np.empty((rows, cols), dtype=np.uint16)
    lib().orc_dequantize(_p(codes, _U8P), _p(scales, _U8P), float(alpha), rows, cols,
                         sf_layout, _p(out32, _F32P), _p(out16, _U16P))
    return out32, out16


def transpose_2d(codes, scales, rows: int, cols: int, sf_layout_in: int = SF_ROWMAJOR,
                 sf_layout_out: int = SF_ROWMAJOR):
    """The encoding of W^T read off a 2D (16x16-tile) encoding of W [rows, cols]:
    returns (codes [cols, rows/2], scales for cols rows x rows/16 blocks)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    out_codes = np.zeros((cols, rows // 2), dtype=np.uint8)
    out_scales = np.zeros(sf_bytes(cols, rows // 16, sf_layout_out), dtype=np.uint8)
    rc = lib().orc_transpose_2d(_p(codes, _U8P), _p(scales, _U8P), rows, cols, sf_layout_in,
                                _p(out_codes, _U8P), _p(out_scales, _U8P), sf_layout_out)
    if rc != 0:
        raise ValueError("bad shape for transpose_2d")
    return out_codes, out_scales


# ---------------------------------------------------------------- GEMM
def gemm(a, b, M: int, N: int, K: int):
    """a, b = (codes, scales, alpha, sf_layout).  Returns (Y, S) fp64 [M, N]."""
    ac, asf, aal, alay = a
    bc, bsf, bal, blay = b
    ac = np.ascontiguousarray(ac, dtype=np.uint8)
    asf = np.ascontiguousarray(asf, dtype=np.uint8)
    bc = np.ascontiguousarray(bc, dtype=np.uint8)
    bsf = np.ascontiguousarray(bsf, dtype=np.uint8)
    y = np.empty((M, N), dtype=np.float64)
    s = np.empty((M, N), dtype=np.float64)
    lib().orc_gemm(_p(ac, _U8P), _p(asf, _U8P), float(aal), alay, _p(bc, _U8P),
                   _p(bsf, _U8P), float(bal), blay, M, N, K, _p(y, _F64P), _p(s, _F64P))
    return y, s


def gemm_pairs(a, b, K: int, mi, ni):
    """Sampled outputs: Y[mi[i], ni[i]] and S for each pair (fp64)."""
    ac, asf, aal, alay = a
    bc, bsf, bal, blay = b
    ac = np.ascontiguousarray(ac, dtype=np.uint8)
    asf = np.ascontiguousarray(asf, dtype=np.uint8)
    bc = np.ascontiguousarray(bc, dtype=np.uint8)
    bsf = np.ascontiguousarray(bsf, dtype=np.uint8)
    mi = np.ascontiguousarray(mi, dtype=np.int64)
    ni = np.ascontiguousarray(ni, dtype=np.int64)
    n = mi.size
    y = np.empty(n, dtype=np.float64)
    s = np.empty(n, dtype=np.float64)
    lib().orc_gemm_pairs(_p(ac, _U8P), _p(asf, _U8P), float(aal), alay, _p(bc, _U8P),
                         _p(bsf, _U8P), float(bal), blay, K, n, _p(mi, _I64P),
                         _p(ni, _I64P), _p(y, _F64P), _p(s, _F64P))
    return y, s
