"""nvfp4_quantize_1d_batched_noalloc: the batched quantizer for callers that
cannot allocate device memory or pass a workspace (a plugin inside another
framework's allocator, a loop that must not synchronize on cudaMalloc, a C
caller holding only its tensors' pointers).  It keeps its amax scratch in a
fixed array inside the library.

Checked through the C ABI against nvfp4_quantize_1d_batched (the entry point
that takes a workspace): codes, scale bytes and global scales must be
identical (bit-exact, as every quantizer test here), on two calls in a row --
the second call must not see the first call's maxima left in the shared
array.  This file is collected last so that a run stopping at the first
failure has run every other test first; it also passes alone."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _descs(xs, outs, capi):
    d = (capi.nvfp4_tensor_desc * len(xs))()
    for i, (x, (codes, scales, alpha)) in enumerate(zip(xs, outs)):
        d[i] = capi.nvfp4_tensor_desc(x.data_ptr(), None, codes.data_ptr(), scales.data_ptr(),
                                      alpha.data_ptr(), x.shape[0], x.shape[1], x.stride(0))
    return d


def _alloc(xs, layout, capi):
    return [(torch.empty((x.shape[0], x.shape[1] // 2), dtype=torch.uint8, device="cuda"),
             torch.empty(capi.nvfp4_scales_bytes(x.shape[0], x.shape[1], layout), dtype=torch.uint8,
                         device="cuda"),
             torch.empty(1, dtype=torch.float32, device="cuda")) for x in xs]


def test_noalloc_matches_workspace_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_block_scaled_20_b200 import build, capi, synth
    build.build()
    stream = torch.cuda.current_stream().cuda_stream
    layout = capi.NVFP4_SF_ROWMAJOR
    qp = capi.nvfp4_qparams(1, 0, 0, 0, layout, 0, None)
    # first call: small-magnitude tensors; second call: larger ones, then
    # small ones again -- a stale max in the shared array would show up as a
    # wrong global scale on the third
    batches = [
        [synth.kv_tensor(3, l, w, heads=4, tokens=48).cuda() * 0.01 for l in range(2) for w in range(2)],
        [synth.kv_tensor(5, l, w, heads=4, tokens=48).cuda() for l in range(2) for w in range(2)],
        [synth.kv_tensor(3, l, w, heads=4, tokens=48).cuda() * 0.01 for l in range(2) for w in range(2)],
    ]
    for xs in batches:
        ref = _alloc(xs, layout, capi)
        ws = torch.zeros(capi.nvfp4_workspace_bytes(len(xs)), dtype=torch.uint8, device="cuda")
        st = capi.nvfp4_quantize_1d_batched(_descs(xs, ref, capi), len(xs), capi.NVFP4_BF16, qp,
                                            ws.data_ptr(), ws.numel(), stream)
        assert st == 0
        got = _alloc(xs, layout, capi)
        st = capi.nvfp4_quantize_1d_batched_noalloc(_descs(xs, got, capi), len(xs),
                                                    capi.NVFP4_BF16, qp, stream)
        assert st == 0
        torch.cuda.synchronize()
        for (rc, rs, ra), (gc, gs, ga) in zip(ref, got):
            assert torch.equal(rc, gc)
            assert torch.equal(rs, gs)
            assert torch.equal(ra, ga)


def test_noalloc_rejects_more_tensors_than_its_scratch():
    from nvfp4_block_scaled_20_b200 import build, capi
    build.build()
    d = (capi.nvfp4_tensor_desc * 65)()
    qp = capi.nvfp4_qparams(1, 0, 0, 0, 0, 0, None)
    assert capi.nvfp4_quantize_1d_batched_noalloc(d, 65, capi.NVFP4_BF16, qp, None) == 2
