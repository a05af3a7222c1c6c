"""The 4-bit Ulysses All-to-All's layout and exchange logic on CPU: two gloo
ranks, each packing its sequence shard of Q ([S_loc * H, d], token-major)
into per-destination NVFP4 segments, exchanging the byte buffers with
all_to_all_single, and dequantizing what arrives.  The encoder and decoder
are the oracle here (the library's kernels need a GPU; the GPU test runs
the same module on them), so this checks the layout, the segment order and
the byte exchange: every rank must end up with the oracle's
quantize-then-dequantize of exactly its heads for the whole sequence, bit
for bit, each (source, destination) segment with its own global scale.
Source: explainer, section 3.4, "The quantization spillover effect"."""
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

S_LOC, HEADS, D, WORLD = 40, 6, 32, 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _full_q():
    """The whole sequence's Q, [WORLD * S_LOC * HEADS, D] token-major bf16."""
    from nvfp4_block_scaled_20_b200 import synth
    return synth.kv_tensor(8, 0, 0, heads=WORLD * S_LOC, tokens=HEADS, head_dim=D)


def _oracle_quantize(xs, outs, stream=None):
    import oracle
    for x, o in zip(xs, outs):
        c, s, a = oracle.quantize_1d(x.float().numpy(), sf_layout=oracle.SF_ROWMAJOR)
        o.codes.copy_(torch.from_numpy(c))
        o.scales.copy_(torch.from_numpy(s))
        o.alpha.copy_(torch.tensor([a], dtype=torch.float32))


def _oracle_dequantize(qs, outs, stream=None):
    import oracle
    for q, o in zip(qs, outs):
        _, b16 = oracle.dequantize(q.codes.numpy(), q.scales.numpy(), float(q.alpha[0]), q.rows,
                                   q.cols, oracle.SF_ROWMAJOR)
        o.view(torch.int16).copy_(torch.from_numpy(b16.view(np.int16)))


def _worker(rank, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    from nvfp4_block_scaled_20_b200 import ulysses
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        full = _full_q()
        shard = full[rank * S_LOC * HEADS:(rank + 1) * S_LOC * HEADS].contiguous()
        layout = ulysses.PayloadLayout(S_LOC, HEADS, D, WORLD)
        out = ulysses.all_to_all_nvfp4(shard, layout, quantize=_oracle_quantize,
                                       dequantize=_oracle_dequantize)
        q.put((rank, out.view(torch.int16).numpy().copy(), layout.buffer_bytes))
    finally:
        dist.destroy_process_group()


def test_two_rank_exchange_matches_the_oracle():
    import oracle
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(WORLD)]
    for p in ps:
        p.start()
    got = dict((r, (o, nb)) for r, o, nb in (q.get(timeout=180) for _ in ps))
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    full = _full_q().float().numpy().reshape(WORLD * S_LOC, HEADS * D)
    hp = HEADS // WORLD
    for r in range(WORLD):
        want = []
        for i in range(WORLD):  # source rank i's tokens, rank r's heads, own global scale
            seg = np.ascontiguousarray(full[i * S_LOC:(i + 1) * S_LOC, r * hp * D:(r + 1) * hp * D])
            c, s, a = oracle.quantize_1d(seg, sf_layout=oracle.SF_ROWMAJOR)
            want.append(oracle.dequantize(c, s, a, S_LOC, hp * D, oracle.SF_ROWMAJOR)[1])
        want = np.concatenate(want).view(np.int16).reshape(-1, D)
        out, nbytes = got[r]
        assert np.array_equal(out, want), "rank %d" % r
        # the payload: 0.5625 bytes per element plus a 16-byte header per segment
        assert nbytes == WORLD * (16 + S_LOC * hp * D * 9 // 16)
