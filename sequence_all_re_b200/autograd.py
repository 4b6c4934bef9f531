"""Autograd pairing of the re-layout (FastVideo API docs, ulysses_a2a
`try_all_to_all_4D`, which hands the call to an autograd function).

The re-layout is a permutation of elements, y = P x, so the gradient of the
input is the inverse permutation of the output gradient: dL/dx = P^-1 dL/dy.
Mode 1 is the inverse of mode 0, so the backward of a mode-m call is a
mode-(1-m) call on the output gradients, run by the same CUDA kernels. This
holds for the single-GPU re-layout of all w slabs (`all_to_all_4d`) and for
one rank's side of the cross-GPU exchange (`peer_all_to_all_4d`), whose
backward is itself an exchange and so is collective like the forward.
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


class UlyssesAllToAll4DPacked(torch.autograd.Function):
    """forward: mode 0 of w head-packed [B, S, T, H, D] slabs (one launch);
    backward: the packed mode 1 of the T*w output gradients."""

    @staticmethod
    def forward(ctx, a2a: UlyssesA2A, chunked: bool, *xs):
        ctx.a2a = a2a
        ctx.chunked = bool(chunked)
        ctx.w = len(xs)
        outs = a2a.run_packed(list(xs), 0, chunked=ctx.chunked)
        ctx.T = len(outs)
        return tuple(o for per_t in outs for o in per_t)

    @staticmethod
    def backward(ctx, *grads):
        ref = next(g for g in grads if g is not None)
        gs = [(g if g is not None else torch.zeros_like(ref)).contiguous() for g in grads]
        per_t = [gs[t * ctx.w:(t + 1) * ctx.w] for t in range(ctx.T)]
        gin = ctx.a2a.run_packed(per_t, 1, chunked=ctx.chunked)
        return (None, None, *gin)


def all_to_all_4d_packed(a2a: UlyssesA2A, xs, chunked: bool = False) -> list:
    """Differentiable mode-0 re-layout of w head-packed slabs [B, S, T, H, D];
    returns T lists of w slabs (see UlyssesA2A.run_packed)."""
    outs = UlyssesAllToAll4DPacked.apply(a2a, bool(chunked), *xs)
    w = len(xs)
    return [list(outs[t * w:(t + 1) * w]) for t in range(len(outs) // w)]


class PeerAllToAll4D(torch.autograd.Function):
    """forward: this rank's mode-`mode` exchange; backward: the inverse-mode exchange
    of the output gradient (every rank runs it, in the same order)."""

    @staticmethod
    def forward(ctx, ex, mode: int, chunked: bool, x):
        ctx.ex = ex
        ctx.mode = int(mode)
        ctx.chunked = bool(chunked)
        return ex.all_to_all_4d(x.detach(), ctx.mode, chunked=ctx.chunked)

    @staticmethod
    def backward(ctx, grad):
        g = ctx.ex.all_to_all_4d(grad.contiguous(), 1 - ctx.mode, chunked=ctx.chunked)
        return None, None, None, g


def peer_all_to_all_4d(ex, x, mode: int, chunked: bool = False):
    """Differentiable cross-GPU exchange of this rank's slab `x` (see
    sequence_all_re_b200.peer.PeerExchange.all_to_all_4d)."""
    return PeerAllToAll4D.apply(ex, int(mode), bool(chunked), x)
