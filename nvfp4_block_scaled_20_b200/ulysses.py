"""4-bit payload for the Ulysses All-to-All of sequence-parallel attention.

In Ulysses sequence parallelism each of P ranks holds a sequence shard of
Q, K and V, [S_loc tokens, H heads, d], and the All-to-All before attention
gives every rank the whole sequence for H / P of the heads.  The pages cast
the runtime Q to NVFP4 before that exchange (K and V are already NVFP4 in the
cache), so the whole payload travels at about 4.5 bits per element instead of
16 and is dequantized on arrival (explainer, section 3.4, "The quantization
spillover effect"; notes, section 3.6, the reading of Figure 8: about 3.6x
less communication).

Layout.  A shard is a token-major [S_loc * H, d] matrix (row t * H + h).  The
heads bound for rank j are the column range [j * H/P * d, (j + 1) * H/P * d)
of the [S_loc, H * d] view, so one descriptor per destination -- rows S_loc,
cols H/P * d, row stride H * d -- quantizes exactly that destination's data
with 16-blocks along d (d is a multiple of 16: the blocks never straddle two
heads), one global scale per (source, destination) segment.  The quantizer
writes each descriptor's codes, scale bytes (row-major) and global scale
straight into that destination's segment of one send buffer:

    segment = [global scale, fp32, padded to 16 bytes | codes | scale bytes]

so the All-to-All moves one contiguous byte buffer with equal splits, and on
the receiving side one batched dequantization turns the P received segments
into the [P * S_loc, H/P, d] bf16 result (segment i = tokens of rank i).

Everything numeric runs in the library's kernels (one batched quantize, one
batched dequantize); this module computes the layout and makes the calls.
The collective is the process group's all_to_all_single (NCCL over NVLink on
B200).  Which encoder and decoder run is a parameter, so the same layout and
exchange logic can be exercised on the host.
"""
from __future__ import annotations

from dataclasses import dataclass

from . import capi


def _pad16(n: int) -> int:
    return (n + 15) // 16 * 16


@dataclass(frozen=True)
class PayloadLayout:
    """Byte layout of one rank's send (or receive) buffer."""
    s_loc: int      # tokens per rank
    heads: int      # H, total heads
    d: int          # head dimension (multiple of 16)
    world: int      # P, ranks

    def __post_init__(self):
        if self.heads % self.world or self.d % 16 or self.s_loc < 0:
            raise ValueError("heads must divide by the world size and d by 16")

    @property
    def heads_per_rank(self) -> int:
        return self.heads // self.world

    @property
    def seg_cols(self) -> int:       # elements per token in one segment
        return self.heads_per_rank * self.d

    @property
    def codes_offset(self) -> int:
        return 16

    @property
    def codes_bytes(self) -> int:
        return _pad16(self.s_loc * self.seg_cols // 2)

    @property
    def scales_offset(self) -> int:
        return self.codes_offset + self.codes_bytes

    @property
    def scales_bytes(self) -> int:
        return _pad16(self.s_loc * self.seg_cols // 16)

    @property
    def segment_bytes(self) -> int:
        return self.scales_offset + self.scales_bytes

    @property
    def buffer_bytes(self) -> int:
        return self.world * self.segment_bytes

    def segment_views(self, buf, j):
        """(codes [s_loc, seg_cols/2], scale bytes [s_loc * seg_cols/16],
        global scale [1] fp32) of segment j, as views of the uint8 buffer."""
        import torch
        base = j * self.segment_bytes
        codes = buf[base + self.codes_offset:base + self.codes_offset
                    + self.s_loc * self.seg_cols // 2].view(self.s_loc, self.seg_cols // 2)
        scales = buf[base + self.scales_offset:base + self.scales_offset
                     + self.s_loc * self.seg_cols // 16]
        alpha = buf[base:base + 4].view(torch.float32)
        return codes, scales, alpha


def _lib_quantize(xs, outs, stream=None):
    import nvfp4_block_scaled_20_b200 as nv
    nv.quantize_1d_batched(xs, sf_layout=capi.NVFP4_SF_ROWMAJOR, outs=outs, stream=stream)


def _lib_dequantize(qs, outs, stream=None):
    import nvfp4_block_scaled_20_b200 as nv
    nv.dequantize(qs, out_dtype=outs[0].dtype, outs=outs, stream=stream)


def pack(x, layout: PayloadLayout, send, quantize=_lib_quantize, stream=None):
    """Quantize this rank's shard x ([s_loc * H, d], token-major) into the
    send buffer (uint8, layout.buffer_bytes): one segment per destination."""
    import nvfp4_block_scaled_20_b200 as nv
    L = layout
    if x.shape != (L.s_loc * L.heads, L.d) or send.numel() < L.buffer_bytes:
        raise ValueError("shard or send buffer does not match the layout")
    xv = x.view(L.s_loc, L.heads * L.d)
    views, outs = [], []
    for j in range(L.world):
        views.append(xv[:, j * L.seg_cols:(j + 1) * L.seg_cols])
        codes, scales, alpha = L.segment_views(send, j)
        outs.append(nv.QTensor(codes, scales, alpha, L.s_loc, L.seg_cols,
                               capi.NVFP4_SF_ROWMAJOR))
    quantize(views, outs, stream=stream)
    return outs


def unpack(recv, layout: PayloadLayout, out, dequantize=_lib_dequantize, stream=None):
    """Dequantize the P received segments into out ([P * s_loc * H/P, d],
    token-major over the whole sequence: segment i holds tokens
    [i * s_loc, (i + 1) * s_loc))."""
    import nvfp4_block_scaled_20_b200 as nv
    L = layout
    if out.shape != (L.world * L.s_loc * L.heads_per_rank, L.d):
        raise ValueError("output does not match the layout")
    ov = out.view(L.world * L.s_loc, L.seg_cols)
    qs, outs = [], []
    for i in range(L.world):
        codes, scales, alpha = L.segment_views(recv, i)
        qs.append(nv.QTensor(codes, scales, alpha, L.s_loc, L.seg_cols, capi.NVFP4_SF_ROWMAJOR))
        outs.append(ov[i * L.s_loc:(i + 1) * L.s_loc])
    dequantize(qs, outs, stream=stream)
    return out


def exchange(send, recv, group=None):
    """The All-to-All of the byte buffers, equal splits (one segment per rank)."""
    import torch.distributed as dist
    dist.all_to_all_single(recv, send, group=group)
    return recv


def all_to_all_nvfp4(x, layout: PayloadLayout, out=None, group=None, send=None, recv=None,
                     quantize=_lib_quantize, dequantize=_lib_dequantize):
    """pack -> All-to-All -> unpack: this rank's shard out, the full sequence
    for this rank's heads back (bf16 unless out says otherwise)."""
    import torch
    dev = x.device
    send = torch.empty(layout.buffer_bytes, dtype=torch.uint8, device=dev) if send is None else send
    recv = torch.empty(layout.buffer_bytes, dtype=torch.uint8, device=dev) if recv is None else recv
    if out is None:
        out = torch.empty((layout.world * layout.s_loc * layout.heads_per_rank, layout.d),
                          dtype=torch.bfloat16, device=dev)
    pack(x, layout, send, quantize)
    exchange(send, recv, group)
    return unpack(recv, layout, out, dequantize)
