"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

This module holds no attention arithmetic.  It only turns a seed into
reproducible bf16 tensors and integer key lengths, so that the fp64 oracle and
the CUDA path see bit-identical inputs.

Generator
---------
* counter-based splitmix64: element ``i`` of stream ``seed`` is
  ``mix(seed * 2**32 + i + 1)`` where ``mix`` is Steele, Lea and Flood's
  splitmix64 finaliser (multiply by the golden-ratio increment, then two
  xor-shift-multiply rounds and a final xor-shift);
* a normal draw uses two uniforms ``u1, u2 in (0, 1]`` (53-bit mantissas) and
  the Box-Muller cosine branch ``sqrt(-2 ln u1) * cos(2 pi u2)``;
* fp64 -> fp32 -> bf16, each step round-to-nearest-even.

The workloads' tensors are i.i.d. N(0, 1) in bf16, laid out ``[B, H, L, d]``
row-major; per-request key lengths are integers uniform in ``[lo, hi]``.
8-bit inputs are those bf16 tensors quantised to E4M3 with one fp32 scale per
128-row tile of each head (the tile's largest magnitude maps to 448).
"""

from __future__ import annotations

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _mix(x: np.ndarray) -> np.ndarray:
    """splitmix64 output function applied to counters ``x`` (uint64, wraps mod 2**64)."""
    with np.errstate(over="ignore"):
        z = x * _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def uniform_u64(seed: int, n: int, offset: int = 0) -> np.ndarray:
    """``n`` raw 64-bit draws of stream ``seed`` starting at counter ``offset``."""
    base = np.uint64((int(seed) & 0xFFFFFFFF) << 32)
    ctr = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(base + ctr)


def _unit(u: np.ndarray) -> np.ndarray:
    """Map raw draws to doubles in (0, 1]."""
    return ((u >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)


def normal_f64(seed: int, n: int) -> np.ndarray:
    """``n`` N(0,1) doubles from stream ``seed`` (Box-Muller, cosine branch)."""
    raw = uniform_u64(seed, 2 * n)
    u1 = _unit(raw[0::2])
    u2 = _unit(raw[1::2])
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 (RNE) -> bf16 (RNE); returns the bf16 bit patterns as uint16."""
    f = np.ascontiguousarray(x, dtype=np.float64).astype(np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    # round-to-nearest-even on the 16 dropped bits; NaN/Inf do not occur here
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    b = (b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return b.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp64."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def normal_bf16(seed: int, shape) -> np.ndarray:
    """i.i.d. N(0,1) tensor of the given shape, as bf16 bit patterns (uint16)."""
    n = int(np.prod(shape)) if len(shape) else 1
    return f64_to_bf16_bits(normal_f64(seed, n)).reshape(shape)


def normal_bf16_block(seed: int, shape, index, first: int = None) -> np.ndarray:
    """``normal_bf16(seed, shape)[index]`` for a tuple ``index`` of leading
    indices (e.g. (b, h) of a [B, H, L, d] tensor), drawn directly at its
    counters: element i of the full tensor uses the stream's draws 2 i and
    2 i + 1, so a block needs no more than its own draws.  ``first``: only the
    block's first ``first`` entries along its leading axis (e.g. rows [0, first))."""
    shape = tuple(int(x) for x in shape)
    index = tuple(int(x) for x in index)
    inner = shape[len(index):]
    n = int(np.prod(inner)) if inner else 1
    if first is not None:
        if not inner or not 0 <= first <= inner[0]:
            raise IndexError("first out of range")
        n_full, inner = n, (int(first),) + inner[1:]
        n = int(np.prod(inner))
    start = 0
    for i, (ix, ext) in enumerate(zip(index, shape)):
        if not 0 <= ix < ext:
            raise IndexError("block index out of range")
        start = start * ext + ix
    start *= n if first is None else n_full
    raw = uniform_u64(seed, 2 * n, offset=2 * start)
    x = np.sqrt(-2.0 * np.log(_unit(raw[0::2]))) * np.cos(2.0 * np.pi * _unit(raw[1::2]))
    return f64_to_bf16_bits(x).reshape(inner)


def uniform_int(seed: int, n: int, lo: int, hi: int) -> np.ndarray:
    """``n`` integers uniform in ``[lo, hi]`` (int32)."""
    raw = uniform_u64(seed, n)
    span = np.uint64(hi - lo + 1)
    return (np.int64(lo) + (raw % span).astype(np.int64)).astype(np.int32)


def to_torch_bf16(bits: np.ndarray):
    """View bf16 bit patterns as a CPU ``torch.bfloat16`` tensor (no copy of values)."""
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def quantize_e4m3_tiles(x, tile: int = 128):
    """Quantise a float32 torch tensor [..., L, d] to E4M3 codes with one scale per
    ``tile`` rows (scale = the tile's largest magnitude / 448, the format's
    largest finite value); the rounding is torch's float8_e4m3fn conversion.
    Returns (codes uint8 [..., L, d], scales float32 [..., ceil(L / tile)]) as
    tensors on x's device."""
    import torch

    L, d = x.shape[-2], x.shape[-1]
    nt = (L + tile - 1) // tile
    lead = x.shape[:-2]
    xp = torch.zeros(*lead, nt * tile, d, dtype=torch.float32, device=x.device)
    xp[..., :L, :] = x
    xt = xp.view(*lead, nt, tile, d)
    amax = xt.abs().amax(dim=(-1, -2))
    scale = torch.clamp(amax, min=2.0 ** -100) / 448.0
    y = torch.clamp(xt / scale[..., None, None], -448.0, 448.0)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8).view(*lead, nt * tile, d)[..., :L, :]
    return codes.contiguous(), scale.contiguous()


def normal_e4m3(seed: int, shape, tile: int = 128):
    """The bf16 N(0,1) tensor of :func:`normal_bf16` quantised per row tile with
    :func:`quantize_e4m3_tiles`; returns numpy (codes uint8, scales float32)."""
    import torch

    x = torch.from_numpy(bf16_bits_to_f64(normal_bf16(seed, shape)).astype(np.float32))
    c, s = quantize_e4m3_tiles(x, tile)
    return c.numpy(), s.numpy()


# Workload seeds: 46 * 100 + workload number; each tensor draws its own stream.
def workload_seed(workload: int, tensor: str) -> int:
    tags = {"q": 1, "k": 2, "v": 3, "do": 4, "klen": 5, "pages": 6}
    return (4600 + workload) * 16 + tags[tensor]


__all__ = [
    "normal_bf16_block",
    "uniform_u64",
    "normal_f64",
    "f64_to_bf16_bits",
    "bf16_bits_to_f64",
    "normal_bf16",
    "quantize_e4m3_tiles",
    "normal_e4m3",
    "uniform_int",
    "to_torch_bf16",
    "workload_seed",
]


# ---------------------------------------------------------------- device-side generation
# The same counter-based splitmix64 + Box-Muller recipe written with torch
# tensor ops, for workloads too large to draw on the host (the decode cache is
# 8.6 GB).  The device's fp64 log/cos may differ from numpy's in the last ulp,
# so the two generators agree except in rare rounding ties; tests of large
# workloads therefore always hand the oracle the bits that were actually used
# (copied back from the device).


def _t_mix(x):
    import torch

    def srl(z, k):  # logical right shift of int64 bit patterns
        return (z >> k) & ((1 << (64 - k)) - 1)

    def c64(v):  # uint64 constant as a wrapped int64
        return v - (1 << 64) if v >= (1 << 63) else v

    z = x * c64(0x9E3779B97F4A7C15)
    z = (z ^ srl(z, 30)) * c64(0xBF58476D1CE4E5B9)
    z = (z ^ srl(z, 27)) * c64(0x94D049BB133111EB)
    return z ^ srl(z, 31)


def normal_bf16_device(seed: int, shape, device, chunk: int = 1 << 25):
    """Device twin of :func:`normal_bf16`: returns a ``torch.bfloat16`` tensor."""
    import torch

    n = int(np.prod(shape)) if len(shape) else 1
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    base = (int(seed) & 0xFFFFFFFF) << 32
    base = base - (1 << 64) if base >= (1 << 63) else base
    for s in range(0, n, chunk):
        m = min(chunk, n - s)
        ctr = torch.arange(2 * s + 1, 2 * (s + m) + 1, dtype=torch.int64, device=device)
        z = _t_mix(ctr + base)
        u = (((z >> 11) & ((1 << 53) - 1)).to(torch.float64) + 1.0) * (2.0 ** -53)
        u1, u2 = u[0::2], u[1::2]
        x = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(2.0 * np.pi * u2)
        out[s:s + m] = x.to(torch.float32).to(torch.bfloat16)
    return out.view(*shape)


def normal_e4m3_device(seed: int, shape, device, tile: int = 128):
    """Device twin of :func:`normal_e4m3` (drawn with :func:`normal_bf16_device`);
    returns torch (codes uint8, scales float32) on ``device``."""
    x = normal_bf16_device(seed, shape, device).float()
    return quantize_e4m3_tiles(x, tile)
