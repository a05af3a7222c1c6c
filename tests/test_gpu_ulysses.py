"""The 4-bit Ulysses payload on the GPU: four sequence-parallel ranks
emulated on one device.  Each rank's Q shard is packed by the library's
batched quantizer straight into its send buffer's per-destination segments;
the All-to-All is emulated by copying segment j of rank r's send buffer to
segment r of rank j's receive buffer (the bytes an all_to_all_single with
equal splits moves); each rank's receive buffer is dequantized by one
batched dequantize.  Every rank's result must equal, bit for bit, the
oracle's quantize-then-dequantize of its heads for the whole sequence, each
(source, destination) segment with its own global scale; and the payload
is 0.5625 bytes per element plus a 16-byte header per segment (explainer,
section 3.4, "The quantization spillover effect": ~4.5 bits instead of 16).
DiT inference shape: 24 heads of 128, SP = 4, 1560 tokens per rank."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_block_scaled_20_b200 import synth, ulysses
from gpu_helpers import DEV, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


@pytest.mark.parametrize("s_loc,heads,d,world", [(1560, 24, 128, 4), (40, 6, 32, 2)])
def test_loopback_exchange_matches_the_oracle(s_loc, heads, d, world):
    L = ulysses.PayloadLayout(s_loc, heads, d, world)
    full = synth.kv_tensor(9, 1, 0, heads=world * s_loc, tokens=heads, head_dim=d)
    shards = [full[r * s_loc * heads:(r + 1) * s_loc * heads].to(DEV) for r in range(world)]
    send = [torch.full((L.buffer_bytes,), 0xEE, dtype=torch.uint8, device=DEV) for _ in shards]
    recv = [torch.empty_like(b) for b in send]
    for x, b in zip(shards, send):
        ulysses.pack(x, L, b)
    seg = L.segment_bytes
    for r in range(world):          # emulated All-to-All
        for j in range(world):
            recv[j][r * seg:(r + 1) * seg].copy_(send[r][j * seg:(j + 1) * seg])
    outs = [ulysses.unpack(recv[j], L, torch.empty((world * s_loc * L.heads_per_rank, d),
                                                   dtype=torch.bfloat16, device=DEV))
            for j in range(world)]
    torch.cuda.synchronize()
    assert L.buffer_bytes == world * (16 + s_loc * L.seg_cols * 9 // 16)
    hf = full.float().numpy().reshape(world * s_loc, heads * d)
    for r in range(world):
        want = []
        for i in range(world):
            blk = np.ascontiguousarray(hf[i * s_loc:(i + 1) * s_loc,
                                          r * L.seg_cols:(r + 1) * L.seg_cols])
            c, s, a = oracle.quantize_1d(blk, sf_layout=oracle.SF_ROWMAJOR)
            # the segment's global scale travelled in its header
            got_a = recv[r][i * seg:i * seg + 4].view(torch.float32).item()
            assert got_a == np.float32(a), (r, i, got_a, a)
            want.append(oracle.dequantize(c, s, a, s_loc, L.seg_cols, oracle.SF_ROWMAJOR)[1])
        want = np.concatenate(want).view(np.int16).reshape(-1, d)
        got = outs[r].view(torch.int16).cpu().numpy()
        assert np.array_equal(got, want), "rank %d: %d elements differ" % (r, (got != want).sum())
