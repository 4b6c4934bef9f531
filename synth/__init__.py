"""Seeded synthetic rank slabs for the Ulysses 4D all-to-all re-layout.

This module only draws numbers. It holds none of the re-layout's arithmetic: it
knows the shape of one rank's slab, a seed and a value distribution, nothing
about how slabs are permuted. Both the CPU oracle's tests and the CUDA path's
tests (and the benchmark) take their inputs from here, so the two sides see the
same bytes.

Recipe (the pages publish no dataset; these stand in for video-DiT activations):
  * one tensor per logical rank, drawn in rank order, rank ``k`` seeded with
    ``seed0 + k`` on a CPU ``torch.Generator``;
  * ``normal``: N(0, 1) drawn as float32, then cast to the target dtype
    (round-to-nearest-even by torch);
  * ``uniform``: U[-1, 1) drawn as float32, then cast;
  * ``unique``: every element of every slab carries a distinct integer id
    (rank-major flat index), so a misplaced element can never match by chance.
"""

from __future__ import annotations

import torch

SEED0 = 1234

_DTYPES = {
    "bf16": torch.bfloat16,
    "fp16": torch.float16,
    "fp32": torch.float32,
    "f32": torch.float32,
    "fp64": torch.float64,
    "u8": torch.uint8,
    "i16": torch.int16,
    "i32": torch.int32,
    "i64": torch.int64,
}


def torch_dtype(name_or_dtype) -> torch.dtype:
    if isinstance(name_or_dtype, torch.dtype):
        return name_or_dtype
    return _DTYPES[name_or_dtype]


def slab_shape(mode: int, w: int, B: int, S_local: int, H: int, D: int) -> tuple:
    """Shape of one rank's *input* slab for ``mode`` (given in mode-0-local terms)."""
    if mode == 0:
        return (B, S_local, H, D)
    return (B, S_local * w, H // w, D)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def normal_slabs(shape, w: int, dtype="bf16", seed0: int = SEED0) -> list:
    """w CPU tensors of ``shape``, N(0,1) float32 cast to ``dtype``."""
    dt = torch_dtype(dtype)
    return [torch.randn(shape, generator=_gen(seed0 + k), dtype=torch.float32).to(dt)
            for k in range(w)]


def uniform_slabs(shape, w: int, dtype="bf16", seed0: int = SEED0) -> list:
    """w CPU tensors of ``shape``, U[-1,1) float32 cast to ``dtype``."""
    dt = torch_dtype(dtype)
    out = []
    for k in range(w):
        u = torch.rand(shape, generator=_gen(seed0 + k), dtype=torch.float32)
        out.append((u * 2.0 - 1.0).to(dt))
    return out


def unique_slabs(shape, w: int, elem_bytes: int) -> list:
    """w CPU integer tensors whose elements are all distinct across all slabs.

    Element value = rank * numel(shape) + flat index within the slab, stored in an
    integer type of ``elem_bytes`` bytes. Raises if the ids do not fit that type.
    """
    numel = 1
    for n in shape:
        numel *= int(n)
    total = numel * w
    dt = {1: torch.uint8, 2: torch.int16, 4: torch.int32, 8: torch.int64}[elem_bytes]
    limit = 1 << (8 * elem_bytes)
    if total > limit:
        raise ValueError(f"{total} ids do not fit {elem_bytes}-byte elements")
    out = []
    for k in range(w):
        ids = torch.arange(k * numel, (k + 1) * numel, dtype=torch.int64)
        if elem_bytes < 8:
            # wrap into the signed storage type: the bit pattern is what counts
            ids = torch.where(ids >= limit // 2, ids - limit, ids)
        out.append(ids.to(dt).reshape(shape))
    return out


def rank_tagged_slabs(shape, w: int) -> list:
    """w int16 CPU tensors: high byte = rank, low byte = flat index mod 256.

    For 2-byte elements on shapes too large for globally unique ids: a position
    holding the wrong rank's element, or an element from the wrong 256-block
    offset, shows up as a mismatch even when the N(0,1) values would collide.
    """
    numel = 1
    for n in shape:
        numel *= int(n)
    out = []
    for k in range(w):
        lo = torch.arange(numel, dtype=torch.int64) % 256
        v = (k << 8) | lo
        v = torch.where(v >= 32768, v - 65536, v)
        out.append(v.to(torch.int16).reshape(shape))
    return out


def random_byte_slabs(shape, w: int, seed0: int = SEED0) -> list:
    """w uint8 CPU tensors of ``shape``, uniform random bytes, rank k seeded seed0+k."""
    return [torch.randint(0, 256, tuple(shape), dtype=torch.uint8, generator=_gen(seed0 + k))
            for k in range(w)]


def poison_like(t: torch.Tensor) -> torch.Tensor:
    """A tensor shaped like ``t`` with every byte 0xFF (an unwritten-output marker)."""
    out = torch.empty_like(t)
    out.view(torch.uint8).fill_(0xFF)
    return out
