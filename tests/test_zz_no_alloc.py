"""nvfp4_quantize_1d_batched_noalloc: the batched quantizer for callers that
cannot allocate device memory or pass a workspace (a plugin inside another
framework's allocator, a loop that must not synchronize on cudaMalloc, a C
caller holding only its tensors' pointers).  It keeps its amax scratch in a
fixed array inside the library.

Checked through the C ABI against nvfp4_quantize_1d_batched (the entry point
that takes a workspace): codes, scale bytes (tcgen05 padding included) and
global scales must be identical (bit-exact, as every quantizer test here),
for both scale layouts, both input dtypes, with and without the fused RHT,
on calls in a row -- a later call must not see an earlier call's maxima left
in the shared array -- and with an empty tensor in the batch.  This file is
collected last so that a run stopping at the first failure has run every
other test first; it also passes alone."""
import ctypes

import pytest
import torch


def _descs(xs, outs, capi):
    d = (capi.nvfp4_tensor_desc * len(xs))()
    for i, (x, (codes, scales, alpha)) in enumerate(zip(xs, outs)):
        d[i] = capi.nvfp4_tensor_desc(x.data_ptr() if x.numel() else None, None,
                                      codes.data_ptr(), scales.data_ptr(), alpha.data_ptr(),
                                      x.shape[0], x.shape[1], x.stride(0))
    return d


def _alloc(xs, layout, capi):
    # at least 16 bytes per buffer so an empty tensor still gets valid, aligned pointers
    return [(torch.full((max(1, x.shape[0]), max(16, x.shape[1] // 2)), 0xA5, dtype=torch.uint8,
                        device="cuda"),
             torch.full((max(16, capi.nvfp4_scales_bytes(x.shape[0], x.shape[1], layout)),), 0xA5,
                        dtype=torch.uint8, device="cuda"),
             torch.full((1,), -1.0, dtype=torch.float32, device="cuda")) for x in xs]


@pytest.mark.gpu
@pytest.mark.parametrize("layout", [0, 1], ids=["rowmajor", "tcgen05"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rht", [0, 1], ids=["plain", "rht"])
def test_noalloc_matches_workspace_entry_point_in_a_row(layout, dtype, rht):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_block_scaled_20_b200 import build, capi, synth
    build.build()
    stream = torch.cuda.current_stream().cuda_stream
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    code = capi.NVFP4_BF16 if dtype == "bf16" else capi.NVFP4_F32
    qp = capi.nvfp4_qparams(1, rht, 0xCDAF if rht else 0, 0, layout, 0, None)

    def kv(seed, scale):
        # 4 tensors of [4 heads * 48 tokens, 128] (a ragged last 128-row atom),
        # and an empty one in the middle of the batch
        xs = [(synth.kv_tensor(seed, l, w, heads=4, tokens=48).cuda().float() * scale).to(tdt)
              for l in range(2) for w in range(2)]
        return xs[:2] + [torch.empty((0, 128), dtype=tdt, device="cuda")] + xs[2:]

    # small magnitudes, then larger ones, then small ones again: a stale max
    # in the shared array would show up as a wrong global scale on the third
    for xs in (kv(3, 0.01), kv(5, 1.0), kv(3, 0.01)):
        ref = _alloc(xs, layout, capi)
        ws = torch.zeros(capi.nvfp4_workspace_bytes(len(xs)), dtype=torch.uint8, device="cuda")
        st = capi.nvfp4_quantize_1d_batched(_descs(xs, ref, capi), len(xs), code, qp,
                                            ws.data_ptr(), ws.numel(), stream)
        assert st == 0
        got = _alloc(xs, layout, capi)
        st = capi.nvfp4_quantize_1d_batched_noalloc(_descs(xs, got, capi), len(xs), code, qp,
                                                    stream)
        assert st == 0
        torch.cuda.synchronize()
        for i, ((rc, rs, ra), (gc, gs, ga)) in enumerate(zip(ref, got)):
            assert torch.equal(rc, gc), "codes of tensor %d" % i
            assert torch.equal(rs, gs), "scales of tensor %d" % i
            assert torch.equal(ra, ga), "global scale of tensor %d" % i
        assert float(got[2][2].item()) == 1.0  # the empty tensor's global scale


def test_noalloc_rejects_more_tensors_than_its_scratch():
    from nvfp4_block_scaled_20_b200 import build, capi
    build.build()
    d = (capi.nvfp4_tensor_desc * 65)()
    qp = capi.nvfp4_qparams(1, 0, 0, 0, 0, 0, None)
    assert capi.nvfp4_quantize_1d_batched_noalloc(d, 65, capi.NVFP4_BF16, qp, None) == 2


def test_noalloc_checks_empty_descriptors_like_the_workspace_call():
    """An empty tensor is still launched (it receives its global scale), so
    its pointers are validated on the host like any other: a misaligned
    global scale is NVFP4_ERR_ALIGN, a missing one NVFP4_ERR_INVALID_ARG, in
    both batched calls.  Rejected before any launch: no GPU needed."""
    from nvfp4_block_scaled_20_b200 import build, capi
    build.build()
    buf = (ctypes.c_uint8 * 256)()
    base = (ctypes.addressof(buf) + 63) // 64 * 64
    qp = capi.nvfp4_qparams(1, 0, 0, 0, 0, 0, None)
    ws = (ctypes.c_uint8 * capi.nvfp4_workspace_bytes(1))()
    for gs, want in ((base + 2, 3), (None, 1)):
        d = (capi.nvfp4_tensor_desc * 1)()
        d[0] = capi.nvfp4_tensor_desc(None, None, base, base + 32, gs, 0, 128, 128)
        assert capi.nvfp4_quantize_1d_batched_noalloc(d, 1, capi.NVFP4_BF16, qp, None) == want
        assert capi.nvfp4_quantize_1d_batched(d, 1, capi.NVFP4_BF16, qp, ctypes.addressof(ws),
                                              len(ws), None) == want
