"""Autograd pairing of the re-layout (FastVideo API docs, ulysses_a2a
`try_all_to_all_4D`, which hands the call to an autograd function).

The re-layout is a permutation of elements, y = P x, so the gradient of the
input is the inverse permutation of the output gradient: dL/dx = P^-1 dL/dy.
Mode 1 is the inverse of mode 0, so the backward of a mode-m call is a
mode-(1-m) call on the output gradients, run by the same CUDA kernels.
"""

from __future__ import annotations

import torch

from . import UlyssesA2A


class UlyssesAllToAll4D(torch.autograd.Function):
    """forward: the mode-`mode` re-layout of w rank slabs; backward: the inverse mode."""

    @staticmethod
    def forward(ctx, a2a: UlyssesA2A, mode: int, chunked: bool, *xs):
        ctx.a2a = a2a
        ctx.mode = int(mode)
        ctx.chunked = bool(chunked)
        ctx.in_shape = tuple(xs[0].shape)
        ctx.in_dtype = xs[0].dtype
        outs = a2a.run(list(xs), ctx.mode, chunked=ctx.chunked)
        return tuple(outs)

    @staticmethod
    def backward(ctx, *grads):
        # an unused output contributes a zero gradient
        ref = next(g for g in grads if g is not None)
        gs = [(g if g is not None else torch.zeros_like(ref)).contiguous() for g in grads]
        gin = ctx.a2a.run(gs, 1 - ctx.mode, chunked=ctx.chunked)
        return (None, None, None, *gin)


def all_to_all_4d(a2a: UlyssesA2A, xs, mode: int, chunked: bool = False) -> list:
    """Differentiable re-layout of the w slabs `xs` (see UlyssesA2A.run)."""
    return list(UlyssesAllToAll4D.apply(a2a, int(mode), bool(chunked), *xs))
