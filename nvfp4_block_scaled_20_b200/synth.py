"""Seeded synthetic inputs shaped like the DiT workloads (no method arithmetic).

This module is the only code the tests, the oracle harness and the bench
share.  It draws numbers; it does not quantize, transform or scale them.

Generator: a counter-based splitmix64.  Value ``i`` of stream ``(seed, sid)``
is ``mix64(key + i * GAMMA)`` with ``key = mix64(seed * 0x100000001B3 + sid)``
(all mod 2^64), where ``mix64`` is the splitmix64 output function.  Uniforms
are ``((r >> 11) + 0.5) * 2^-53`` in (0, 1); normals come from Box-Muller on
consecutive pairs, in float64; Student-t(3) is ``z0 / sqrt((z1^2+z2^2+z3^2)/3)``
with four independent normal streams.  Outputs are rounded to fp32, then (for
bf16 tensors) to bf16 round-to-nearest-even by torch.  Everything is torch
and runs on the CPU or on a CUDA device; transcendental functions may differ
in the last bit between the two, so a test that needs the same input on both
sides generates it once and copies it.

Recipes (sizes are the workloads'; tests also call them at reduced sizes):
  * activation: N(0, 1), with a seeded Fisher-Yates choice of ``n_out``
    columns either scaled (tiny case: x20) or replaced by Student-t(3) x 8
    ("heavy-tailed channels").
  * weight: N(0, 0.02) (second parameter is the standard deviation).
  * KV: N(0, 1) plus one N(0, 2) scalar per (layer, K/V, head).
  * dY: N(0, 1e-3).
  * RHT sign mask: low 16 bits of splitmix64's first output for a seed.
"""
from __future__ import annotations

import math

import torch

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
_C1 = 0xBF58476D1CE4E5B9
_C2 = 0x94D049BB133111EB
_CHUNK = 1 << 24


def _s64(v: int) -> int:
    v &= MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def mix64_int(z: int) -> int:
    """splitmix64 output function on a Python int (mod 2^64)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * _C1) & MASK64
    z = ((z ^ (z >> 27)) * _C2) & MASK64
    return z ^ (z >> 31)


def _lsr(z: torch.Tensor, k: int) -> torch.Tensor:
    return (z >> k) & ((1 << (64 - k)) - 1)


def _mix64(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _lsr(z, 30)) * _s64(_C1)
    z = (z ^ _lsr(z, 27)) * _s64(_C2)
    return z ^ _lsr(z, 31)


def stream_key(seed: int, sid: int) -> int:
    return mix64_int(seed * 0x100000001B3 + sid)


def raw64(seed: int, sid: int, start: int, n: int, device="cpu") -> torch.Tensor:
    """Counter values start .. start+n-1 of a stream, as int64 bit patterns."""
    key = stream_key(seed, sid)
    idx = torch.arange(start, start + n, dtype=torch.int64, device=device)
    return _mix64(idx * _s64(GAMMA) + _s64(key))


def uniform(seed: int, sid: int, n: int, device="cpu", start: int = 0) -> torch.Tensor:
    r = raw64(seed, sid, start, n, device)
    return (_lsr(r, 11).to(torch.float64) + 0.5) * (2.0 ** -53)


def normal(seed: int, sid: int, n: int, device="cpu") -> torch.Tensor:
    """n standard normals (float64), Box-Muller on pairs of uniforms."""
    out = torch.empty(n, dtype=torch.float64, device=device)
    npairs = (n + 1) // 2
    for p0 in range(0, npairs, _CHUNK):
        p1 = min(npairs, p0 + _CHUNK)
        u = uniform(seed, sid, 2 * (p1 - p0), device, start=2 * p0)
        u1, u2 = u[0::2], u[1::2]
        rad = torch.sqrt(-2.0 * torch.log(u1))
        ang = (2.0 * math.pi) * u2
        z = torch.stack((rad * torch.cos(ang), rad * torch.sin(ang)), dim=1).reshape(-1)
        lo, hi = 2 * p0, min(n, 2 * p1)
        out[lo:hi] = z[: hi - lo]
    return out


def normal_at(seed: int, sid: int, idx: torch.Tensor) -> torch.Tensor:
    """normal(seed, sid, n)[idx] for an index tensor, without drawing the rest:
    element i is one half of the Box-Muller pair i // 2 (uniforms 2 (i // 2)
    and 2 (i // 2) + 1 of the stream)."""
    key = _s64(stream_key(seed, sid))
    pair = idx // 2
    r1 = _mix64((2 * pair) * _s64(GAMMA) + key)
    r2 = _mix64((2 * pair + 1) * _s64(GAMMA) + key)
    u1 = (_lsr(r1, 11).to(torch.float64) + 0.5) * (2.0 ** -53)
    u2 = (_lsr(r2, 11).to(torch.float64) + 0.5) * (2.0 ** -53)
    rad = torch.sqrt(-2.0 * torch.log(u1))
    ang = (2.0 * math.pi) * u2
    return torch.where(idx % 2 == 0, rad * torch.cos(ang), rad * torch.sin(ang))


def student_t3(seed: int, sid: int, n: int, device="cpu") -> torch.Tensor:
    z0 = normal(seed, sid * 4 + 0x10000, n, device)
    chi = normal(seed, sid * 4 + 0x10001, n, device) ** 2
    chi += normal(seed, sid * 4 + 0x10002, n, device) ** 2
    chi += normal(seed, sid * 4 + 0x10003, n, device) ** 2
    return z0 / torch.sqrt(chi / 3.0)


def choose_columns(seed: int, sid: int, ncols: int, k: int) -> list[int]:
    """First k entries of a seeded Fisher-Yates permutation of range(ncols)."""
    perm = list(range(ncols))
    u = uniform(seed, sid, max(ncols - 1, 1)).tolist()
    for t, i in enumerate(range(ncols - 1, 0, -1)):
        j = int(u[t] * (i + 1))
        perm[i], perm[j] = perm[j], perm[i]
    return sorted(perm[:k])


def rht_sign_mask(seed: int = 0) -> int:
    """16 random signs for the Hadamard transform: bit j set means s_j = -1."""
    return mix64_int(seed + GAMMA) & 0xFFFF


def _finish(x64: torch.Tensor, rows: int, cols: int, dtype) -> torch.Tensor:
    x = x64.to(torch.float32).reshape(rows, cols)
    return x if dtype == torch.float32 else x.to(dtype)


def weight(seed: int, sid: int, rows: int, cols: int, dtype=torch.bfloat16,
           std: float = 0.02, device="cpu") -> torch.Tensor:
    return _finish(normal(seed, sid, rows * cols, device) * std, rows, cols, dtype)


def activation(seed: int, sid: int, rows: int, cols: int, dtype=torch.bfloat16,
               n_out: int | None = None, mode: str = "student_t", factor: float = 8.0,
               std: float = 1.0, device="cpu") -> torch.Tensor:
    """N(0, std) with n_out outlier columns (default: ceil(1% of cols)).

    mode "student_t": the columns are replaced by Student-t(3) * factor;
    mode "scale": the columns are multiplied by factor.
    """
    x = normal(seed, sid, rows * cols, device).reshape(rows, cols) * std
    if n_out is None:
        n_out = math.ceil(0.01 * cols)
    if n_out > 0:
        cols_sel = torch.tensor(choose_columns(seed, sid + 0x5000, cols, n_out),
                                dtype=torch.int64, device=device)
        if mode == "scale":
            x[:, cols_sel] *= factor
        else:
            t = student_t3(seed, sid, rows * n_out, device).reshape(rows, n_out)
            x[:, cols_sel] = t * factor
    return _finish(x.reshape(-1), rows, cols, dtype)


def activation_cols(seed: int, sid: int, rows: int, cols: int, c0: int, c1: int,
                    dtype=torch.bfloat16, n_out: int | None = None, factor: float = 8.0,
                    std: float = 1.0) -> torch.Tensor:
    """activation(seed, sid, rows, cols, ...)[:, c0:c1] (mode "student_t"),
    drawn on the host without the other columns."""
    r = torch.arange(rows, dtype=torch.int64)[:, None]
    c = torch.arange(c0, c1, dtype=torch.int64)[None, :]
    x = normal_at(seed, sid, (r * cols + c).reshape(-1)).reshape(rows, c1 - c0) * std
    if n_out is None:
        n_out = math.ceil(0.01 * cols)
    if n_out > 0:
        sel = choose_columns(seed, sid + 0x5000, cols, n_out)
        hit = [(j, col) for j, col in enumerate(sel) if c0 <= col < c1]
        if hit:
            t = student_t3(seed, sid, rows * n_out).reshape(rows, n_out)
            for j, col in hit:
                x[:, col - c0] = t[:, j] * factor
    return _finish(x.reshape(-1), rows, c1 - c0, dtype)


def kv_tensor(seed: int, layer: int, which: int, heads: int = 24, tokens: int = 32760,
              head_dim: int = 128, device="cpu") -> torch.Tensor:
    """One layer's K (which=0) or V (which=1): [heads * tokens, head_dim] bf16,
    N(0, 1) plus a per-head N(0, 2) bias."""
    sid = 0x100 + 2 * layer + which
    x = normal(seed, sid, heads * tokens * head_dim, device).reshape(heads, tokens * head_dim)
    bias = normal(seed, sid + 0x8000, heads, device) * 2.0
    x += bias[:, None]
    return _finish(x.reshape(-1), heads * tokens, head_dim, torch.bfloat16)


# ---------------------------------------------------------------- workloads
def tiny_linear(device="cpu"):
    """X fp32 [64, 256] N(0,1) with 4 columns x20; W fp32 [128, 256] N(0,0.02)."""
    x = activation(0, 1, 64, 256, torch.float32, n_out=4, mode="scale", factor=20.0,
                   device=device)
    w = weight(0, 2, 128, 256, torch.float32, device=device)
    return x, w


def qkv_linear(device="cpu", m: int = 2640, n: int = 9216, k: int = 3072):
    """X bf16 [m, k] (1% Student-t(3) x 8 channels); W bf16 [n, k] N(0, 0.02)."""
    return (activation(1, 1, m, k, device=device),
            weight(1, 2, n, k, device=device))


def ffn_pair(device="cpu", m: int = 8192, d: int = 3072, h: int = 14336):
    """X bf16 [m, d]; W_up [h, d]; W_dn [d, h] (N(0, 0.02))."""
    return (activation(2, 1, m, d, device=device),
            weight(2, 2, h, d, device=device),
            weight(2, 3, d, h, device=device))


def wgrad(device="cpu", t: int = 32768, dout: int = 3072, din: int = 14336):
    """dY bf16 [t, dout] N(0, 1e-3); X bf16 [t, din] with outlier channels."""
    dy = activation(4, 1, t, dout, n_out=0, std=1e-3, device=device)
    x = activation(4, 2, t, din, device=device)
    return dy, x, rht_sign_mask(0)
