"""Failure detection on the device: a bounded GEMM wait that runs out is
reported, and the device stays usable.

The test makes a wait run out on purpose without any fault: with the test
hook on (nvfp4_set_test_stall), every GEMM's MMA issuer first waits, bounded
by nvfp4_set_wait_limit, on a barrier nothing ever completes, while the
producers' first stages of tile loads are in flight.  The kernel must then
record NVFP4_ERR_TIMEOUT in the workspace error word (read back by
nvfp4_get_device_error), wait for every copy and MMA it issued, free its
tensor memory and return; the next GEMM on the same device must give the
oracle's result with no error recorded."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_block_scaled_20_b200 as nv
from nvfp4_block_scaled_20_b200 import capi, synth
from gpu_helpers import DEV, gemm_tolerance, require_gpu, to_oracle

pytestmark = pytest.mark.gpu

NVFP4_ERR_TIMEOUT = 6


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def test_gemm_wait_that_runs_out_is_reported_and_the_device_stays_usable():
    M, N, K = 512, 768, 4096  # 2 x 3 tiles of 256 x 256, 16 stages each
    x = synth.activation(70, 1, M, K)
    w = synth.weight(70, 2, N, K)
    qa = nv.quantize_1d(x.to(DEV))
    qb = nv.quantize_2d(w.to(DEV))
    ws = nv.workspace(0)
    out = torch.full((M, N), 7.0, dtype=torch.float32, device=DEV)
    try:
        assert capi.nvfp4_set_wait_limit(2_000_000) == 0  # 2 ms
        assert capi.nvfp4_set_test_stall(1) == 0
        nv.gemm(qa, qb, out=out, ws=ws)
        torch.cuda.synchronize()
    finally:
        capi.nvfp4_set_test_stall(0)
        capi.nvfp4_set_wait_limit(0)
    assert nv.device_error(ws) == NVFP4_ERR_TIMEOUT
    assert nv.device_error(ws) == 0  # read back once, then cleared

    # the device is still usable: the same GEMM now completes, in tolerance
    nv.gemm(qa, qb, out=out, ws=ws)
    torch.cuda.synchronize()
    assert nv.device_error(ws) == 0
    aref = oracle.quantize_1d(to_oracle(x), sf_layout=oracle.SF_TCGEN05)
    bref = oracle.quantize_2d(to_oracle(w), sf_layout=oracle.SF_TCGEN05)
    y, s = oracle.gemm((aref[0], aref[1], aref[2], oracle.SF_TCGEN05),
                       (bref[0], bref[1], bref[2], oracle.SF_TCGEN05), M, N, K)
    got = out.cpu().numpy().astype(np.float64)
    assert (np.abs(got - y) <= gemm_tolerance(y, s, False)).all()


def test_test_hook_arguments():
    assert capi.nvfp4_set_test_stall(2) == 1
    assert capi.nvfp4_set_test_stall(0) == 0
    assert capi.nvfp4_set_wait_limit(0) == 0
