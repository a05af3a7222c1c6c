"""Exhaustive sweeps of the two hardware conversions every encoder takes its
rounding decisions with (cvt.rn.satfinite.e2m1x2.f32 for element codes,
cvt.rn.satfinite.e4m3x2.f32 for scale codes), through nvfp4_convert_sweep,
against the oracle's casts -- the pages' "rounded to the nearest E2M1
value" and "cast_E4M3 ... nearest representable E4M3 value" (explainer,
"Quantization rule for a tensor block") under the readings ties-to-even and
saturation at 6 / 448.

E2M1: every fp32 of magnitude below 16, both signs (an encoder's quotient
y / s stays below 9: the scale codes round the block maximum's quotient to
at most 6 * 1.5 in the subnormal scale range).  E4M3: every non-negative
fp32, +inf included (candidate scales are non-negative).  About 4.3e9
inputs in all, compared in chunks on the host pool."""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_20_b200 import capi
from gpu_helpers import DEV, require_gpu

pytestmark = pytest.mark.gpu

try:
    _THREADS = max(1, len(os.sched_getaffinity(0)))
except AttributeError:  # pragma: no cover
    _THREADS = max(1, os.cpu_count() or 1)

_CHUNK = 1 << 27


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def sweep(target: int, first: int, last: int):
    """GPU conversions of bit patterns [first, last) against the oracle's,
    chunk by chunk; returns the number of inputs checked."""
    buf = torch.empty(_CHUNK, dtype=torch.uint8, device=DEV)
    stream = torch.cuda.current_stream().cuda_stream
    bad = []
    with ThreadPoolExecutor(max_workers=_THREADS) as ex:
        for c0 in range(first, last, _CHUNK):
            n = min(_CHUNK, last - c0)
            assert capi.nvfp4_convert_sweep(target, c0, n, buf.data_ptr(), stream) == 0
            got = buf[:n].cpu().numpy()
            part = -(-n // _THREADS)

            def cmp(p0):
                p1 = min(n, p0 + part)
                want = oracle.encode_bits(target, c0 + p0, p1 - p0)
                idx = np.nonzero(got[p0:p1] != want)[0]
                return [(c0 + p0 + int(i), int(got[p0 + i]), int(want[i])) for i in idx[:5]]

            for r in ex.map(cmp, range(0, n, part)):
                bad += r
            if len(bad) > 20:
                break
    assert not bad, "first mismatches (bits, gpu, oracle): " + ", ".join(
        "(0x%08x, 0x%02x, 0x%02x)" % b for b in bad[:10])
    return last - first


def test_e2m1_conversion_every_input_below_16():
    n = sweep(0, 0x00000000, 0x41800000)        # +0 .. just below +16
    n += sweep(0, 0x80000000, 0xC1800000)       # -0 .. just above -16
    assert n == 2 * 0x41800000


def test_e4m3_conversion_every_non_negative_input():
    n = sweep(1, 0x00000000, 0x7F800001)        # +0 .. +inf
    assert n == 0x7F800001
