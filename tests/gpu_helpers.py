"""Shared helpers for the -m gpu parity tests: run the CUDA path through the
C ABI and the oracle on the same seeded inputs, compare."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_block_scaled_20_b200 as nv
from nvfp4_block_scaled_20_b200 import build

DEV = "cuda"


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def to_oracle(x: torch.Tensor) -> np.ndarray:
    """Generator output (CPU tensor, bf16 or fp32) widened exactly to fp32."""
    return x.detach().to("cpu").to(torch.float32).numpy()


def mismatch_report(got: np.ndarray, want: np.ndarray, what: str, limit: int = 10) -> str:
    bad = np.nonzero(got.reshape(-1) != want.reshape(-1))[0]
    if bad.size == 0:
        return ""
    lines = ["%s: %d mismatches of %d" % (what, bad.size, got.size)]
    for i in bad[:limit]:
        lines.append("  [%d] gpu=%r oracle=%r" % (i, got.reshape(-1)[i], want.reshape(-1)[i]))
    return "\n".join(lines)


def assert_q_equal(q: nv.QTensor, ref, what=""):
    codes, scales, alpha = ref
    gc = q.codes.cpu().numpy()
    gs = q.scales.cpu().numpy()
    ga = float(q.alpha.cpu()[0])
    msg = mismatch_report(gc, codes, what + " codes") + mismatch_report(gs, scales, what + " scales")
    assert ga == np.float32(alpha), "%s alpha gpu=%r oracle=%r" % (what, ga, alpha)
    assert not msg, msg


def gemm_tolerance(ref_y, ref_s, out_bf16: bool, gelu: bool = False):
    """|gpu - oracle| <= 1e-3 * S with S = sum_k |a_k b_k| (the stated GEMM
    bound), plus half a bf16 ulp of the reference for bf16 outputs.

    With the GELU epilogue the GPU applies GELU to its own accumulator y^,
    |y^ - y| <= 1e-3 S.  GELU-tanh's slope stays below 1.13, so the exact
    GELU of y^ is within 1.13e-3 S of the oracle's GELU(y); the epilogue's own
    evaluation of GELU (tanh from exp) is within 2^-17 |y^| of the exact one
    (derivation beside the device code), and |y^| <= 1.001 S, so 2^-16 S
    covers it."""
    tol = 1e-3 * ref_s
    if gelu:
        tol = 1.13e-3 * ref_s + 2.0 ** -16 * ref_s
    if out_bf16:
        mag = np.abs(ref_y)
        e = np.floor(np.log2(np.where(mag > 0, mag, 1e-300)))
        half_ulp = np.where(mag > 0, 2.0 ** (e - 8), 0.0)
        tol = tol + half_ulp
    return tol


def oracle_gemm_ref(aq, bq, M, N, K, mi=None, ni=None):
    A = (aq[0], aq[1], aq[2], oracle.SF_TCGEN05)
    B = (bq[0], bq[1], bq[2], oracle.SF_TCGEN05)
    if mi is None:
        return oracle.gemm(A, B, M, N, K)
    return oracle.gemm_pairs(A, B, K, mi, ni)
