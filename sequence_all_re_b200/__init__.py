"""B200-native Ulysses 4D all-to-all re-layout.

All ``w`` logical rank slabs live in one GPU's memory, so the Ulysses
all-to-all is a pure permutation (FastVideo API docs,
device_communicators/ulysses_a2a, ``run_armed``):

* mode 0 scatters heads and gathers sequence: each rank's ``[B, S_local, H, D]``
  becomes ``[B, S_local*w, H//w, D]`` with
  ``out_r[b, j*S_local+s, h', d] = x_j[b, s, r*(H//w)+h', d]``;
* mode 1 is the exact inverse;
* ``chunked=True`` runs one launch per batch plane, in stream order;
  ``chunked=2`` stages each plane through a context-owned window first.

The work happens in ``libulysses_a2a.so`` (hand-written CUDA for sm_100a,
C ABI in ``include/ulysses_a2a.h``). This package only marshals tensors into
that ABI; PyTorch supplies device memory and streams. There is no CPU or
PyTorch fallback: if the library is missing, importing this package fails.
"""

from __future__ import annotations

import torch

from . import _lib
from ._lib import A2AError, PATH_AUTO, PATH_STAGED, PATH_TMA, PATH_VEC  # noqa: F401

# torch's current stream as a raw handle (the public torch.cuda.current_stream
# wraps the same handle in a Stream object)
_raw_current_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)

__all__ = ["UlyssesA2A", "BoundRun", "A2AError", "output_shape", "mode0_local_tuple",
           "marshal_slabs", "PATH_AUTO", "PATH_TMA", "PATH_VEC", "PATH_STAGED"]


def output_shape(in_shape, mode: int, w: int) -> tuple:
    """Output slab shape for an input slab shape, as ``run_armed`` derives it."""
    if mode == 0:
        B, S_local, H, D = in_shape
        return (B, S_local * w, H // w, D)
    B, S_global, H_local, D = in_shape
    return (B, S_global // w, H_local * w, D)


def mode0_local_tuple(in_shape, mode: int, w: int) -> tuple:
    """(B, S_local, H, D) handed to the native op in either mode."""
    if mode == 0:
        return tuple(int(v) for v in in_shape)
    B, S_global, H_local, D = in_shape
    return (int(B), int(S_global) // w, int(H_local) * w, int(D))


def row_pitch(ts, allow_pitch: bool) -> int:
    """Row pitch (elements) shared by [B, S, H, D] tensors: 0 when contiguous,
    else p for views whose strides are (S*p, p, D, 1) with p >= H*D (for
    example q, k or v of a packed [B, S, 3, H, D] projection output)."""
    if all(t.is_contiguous() for t in ts):
        return 0
    if not allow_pitch:
        raise ValueError("rank slabs must be contiguous")
    B, S, H, D = ts[0].shape
    pitch = None
    for t in ts:
        st = t.stride()
        p = st[1]
        ok = st[3] == 1 and (H == 1 or st[2] == D) and p >= H * D and (B == 1 or st[0] == S * p)
        if not ok or (pitch is not None and p != pitch):
            raise ValueError("a [B, S, H, D] slab must be contiguous or a view with strides "
                             "(S*p, p, D, 1), p >= H*D, shared by all slabs")
        pitch = p
    return pitch


def marshal_slabs(xs, mode: int, out, device_type: str, elem_bytes: int,
                  allow_pitch: bool = False):
    """Checks one call's slabs and turns them into the C ABI's arguments.

    Returns (w, (B, S_local, H, D), out, input pointers, output pointers, row
    pitch of the [B, S, H, D] side in elements, 0 when contiguous), allocating
    the outputs when ``out`` is None; raises ValueError on slabs the op cannot
    take. One pass over each list, reading only cheap tensor attributes: this
    runs on every call, and on small launches its cost is of the kernel's
    order. Whether each pointer lies in the context device's memory, inside
    its allocation, the library checks itself."""
    w = len(xs)
    if w < 1:
        raise ValueError("need at least one rank slab")
    if mode != 0 and mode != 1:
        raise ValueError("mode must be 0 or 1")
    x0 = xs[0]
    shape, dt = x0.shape, x0.dtype
    if len(shape) != 4:
        raise ValueError("rank slabs are 4D")
    if x0.element_size() != elem_bytes:
        raise ValueError(f"context handles {elem_bytes}-byte elements")
    cuda = device_type == "cuda"
    in_ptrs, in_dense = [], True
    for t in xs:
        if t.shape != shape or t.dtype != dt:
            raise ValueError("rank slabs must share shape and dtype")
        if t.is_cuda != cuda or (not cuda and t.device.type != device_type):
            raise ValueError(f"rank slabs must be on {device_type}")
        in_dense = in_dense and t.is_contiguous()
        in_ptrs.append(t.data_ptr())
    B, S, H, D = mode0_local_tuple(shape, mode, w)
    oshape = output_shape(shape, mode, w)
    if out is None:
        kw = {"dtype": dt, "device": x0.device}
        if not cuda:
            kw["pin_memory"] = x0.is_pinned()
        out = [torch.empty(oshape, **kw) for _ in range(w)]
    elif len(out) != w:
        raise ValueError("need one output per rank")
    out_ptrs, out_dense = [], True
    for o in out:
        if o.shape != oshape or o.dtype != dt:
            raise ValueError(f"outputs must be {oshape} {dt}")
        out_dense = out_dense and o.is_contiguous()
        out_ptrs.append(o.data_ptr())
    # the [B, S, H, D] side (inputs in mode 0, outputs in mode 1) may be pitched
    strided, strided_dense, dense = ((xs, in_dense, out_dense) if mode == 0
                                     else (out, out_dense, in_dense))
    if not dense:
        raise ValueError("the [B, S_local*w, H/w, D] slabs must be contiguous")
    pitch = 0 if strided_dense else row_pitch(strided, allow_pitch)
    return w, (B, S, H, D), out, in_ptrs, out_ptrs, pitch


class BoundRun:
    """One ``UlyssesA2A.run`` call whose arguments were checked and marshalled
    when it was bound (``UlyssesA2A.bind``); calling it launches the re-layout
    on ``stream`` (default: torch's current stream) and returns the outputs."""

    def __init__(self, a2a, xs, out, in_ptrs, out_ptrs, dims, w, mode, chunked, pitch):
        self._a2a = a2a
        self._slabs = xs + list(out)
        self._ptrs = in_ptrs + out_ptrs
        self.out = out
        self._desc = _lib.DescBuffer(max(len(in_ptrs), len(out_ptrs)))
        B, S, H, D = dims
        self._ref = self._desc.fill(in_ptrs, out_ptrs, B, S, H, D, w, mode, chunked, pitch)

    def __call__(self, stream=None):
        for t, ptr in zip(self._slabs, self._ptrs):
            if t.data_ptr() != ptr:
                raise ValueError("a bound slab was reallocated since bind(); bind again")
        a2a = self._a2a
        a2a._check(_lib.run_ex_ref(a2a._ctx, self._ref, a2a._stream_handle(stream)))
        return self.out


class UlyssesA2A:
    """A library context bound to one CUDA device and one element size."""

    def __init__(self, device=0, elem_bytes: int = 2):
        dev = torch.device("cuda", device) if isinstance(device, int) else torch.device(device)
        self.device = dev
        self.elem_bytes = int(elem_bytes)
        self._device_index = dev.index or 0
        self._desc = _lib.DescBuffer()
        self._ctx = _lib.ulysses_a2a_create(dev.index or 0, self.elem_bytes)

    # ------------------------------------------------------------------ knobs
    def set_path(self, path: int) -> None:
        self._check(_lib.ulysses_a2a_set_path(self._ctx, path))

    def set_tuning(self, rows_per_tile: int = 0, ctas_per_sm: int = 0, stages: int = 0,
                   **knobs) -> None:
        """Speed knobs for later runs (see ``ulysses_a2a_tuning_t``); no argument
        restores every default. Extra knobs: lookahead, producers, order, chunk_units."""
        self._check(_lib.ulysses_a2a_set_tuning(self._ctx, rows_per_tile=rows_per_tile,
                                                ctas_per_sm=ctas_per_sm, stages=stages, **knobs))

    def settings(self):
        """(forced path, tuning knobs) of this context, as the library holds them."""
        rc, path, knobs = _lib.ulysses_a2a_get_settings(self._ctx)
        self._check(rc)
        return path, knobs

    @property
    def launch_count(self) -> int:
        return _lib.ulysses_a2a_launch_count(self._ctx)

    def last_error(self) -> str:
        return _lib.ulysses_a2a_last_error(self._ctx)

    def _check(self, rc: int) -> None:
        if rc != _lib.OK:
            raise A2AError(rc, self.last_error())

    # ------------------------------------------------------------- the op
    def _stream_handle(self, stream) -> int:
        """cudaStream_t of ``stream`` (a torch stream or a raw handle); None is
        torch's current stream on this context's device, read without building
        a Stream object (that costs microseconds per call)."""
        if stream is None:
            if _raw_current_stream is not None:
                return _raw_current_stream(self._device_index)
            return torch.cuda.current_stream(self.device).cuda_stream
        return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)

    def run(self, xs, mode: int, chunked: bool = False, out=None, stream=None):
        """Re-layout device slabs ``xs`` (list of w tensors); returns the w outputs.

        The [B, S_local, H, D] side (``xs`` in mode 0, ``out`` in mode 1) may be
        a row-pitched view, e.g. ``qkv[:, :, 0]`` of a packed [B, S, 3, H, D]
        projection output: it is read or written in place. Asynchronous on
        ``stream`` (default: torch's current stream on the device).
        """
        w, (B, S, H, D), out, ip, op, pitch = marshal_slabs(xs, mode, out, "cuda", self.elem_bytes,
                                                            allow_pitch=True)
        ref = self._desc.fill(ip, op, B, S, H, D, w, mode, int(chunked), pitch)
        self._check(_lib.run_ex_ref(self._ctx, ref, self._stream_handle(stream)))
        return out

    def bind(self, xs, mode: int, chunked: bool = False, out=None) -> "BoundRun":
        """``run`` with its slabs checked and marshalled once, for callers that
        re-lay out the same buffers call after call: the returned object's
        ``__call__(stream=None)`` re-reads only the slabs' data pointers (a slab
        reallocated since, by ``resize_`` or ``set_``, raises) and launches.
        The object keeps the slabs alive; their contents may change freely."""
        w, dims, out, ip, op, pitch = marshal_slabs(xs, mode, out, "cuda", self.elem_bytes,
                                                    allow_pitch=True)
        return BoundRun(self, list(xs), out, ip, op, dims, w, mode, int(chunked), pitch)

    def run_packed(self, xs, mode: int, chunked: bool = False, out=None, stream=None):
        """Re-layout T tensors packed along the head dimension in one launch.

        mode 0: ``xs`` is w contiguous tensors [B, S_local, T, H, D] (for example
        a packed q/k/v projection output per rank); returns T lists of w
        tensors [B, S_local*w, H//w, D] (list t holds tensor t of every rank).
        mode 1: ``xs`` is T lists of w tensors [B, S_local*w, H//w, D]; returns
        w tensors [B, S_local, T, H, D]. Same bytes as T calls of ``run`` on
        the per-tensor views; one kernel launch (VEC path).
        """
        if mode not in (0, 1):
            raise ValueError("mode must be 0 or 1")
        if mode == 0:
            w = len(xs)
            if w < 1 or xs[0].dim() != 5:
                raise ValueError("mode 0 takes w tensors [B, S_local, T, H, D]")
            B, S, T, H, D = (int(v) for v in xs[0].shape)
            if H % w:
                raise ValueError("H must be divisible by w")
            ins = list(xs)
            shape_out = (B, S * w, H // w, D)
            if out is None:
                out = [[torch.empty(shape_out, dtype=xs[0].dtype, device=xs[0].device)
                        for _ in range(w)] for _ in range(T)]
            flat_out = [o for per_t in out for o in per_t]
            checks = [(t, (B, S, T, H, D)) for t in ins] + [(o, shape_out) for o in flat_out]
        else:
            T = len(xs)
            w = len(xs[0]) if T else 0
            if T < 1 or w < 1 or xs[0][0].dim() != 4:
                raise ValueError("mode 1 takes T lists of w tensors [B, S_local*w, H/w, D]")
            B, Sg, Hw, D = (int(v) for v in xs[0][0].shape)
            if Sg % w:
                raise ValueError("S_local*w must be divisible by w")
            S, H = Sg // w, Hw * w
            ins = [x for per_t in xs for x in per_t]
            if out is None:
                out = [torch.empty((B, S, T, H, D), dtype=ins[0].dtype, device=ins[0].device)
                       for _ in range(w)]
            flat_out = list(out)
            checks = [(t, (B, Sg, Hw, D)) for t in ins] + [(o, (B, S, T, H, D)) for o in flat_out]
        for t, shape in checks:
            if (tuple(t.shape) != shape or t.dtype != ins[0].dtype or t.device.type != "cuda"
                    or not t.is_contiguous() or t.element_size() != self.elem_bytes):
                raise ValueError(f"every slab must be a contiguous {shape} CUDA tensor of "
                                 f"{self.elem_bytes}-byte elements")
        ref = self._desc.fill([t.data_ptr() for t in ins], [o.data_ptr() for o in flat_out],
                              B, S, H, D, w, mode, int(chunked), 0, T)
        self._check(_lib.run_ex_ref(self._ctx, ref, self._stream_handle(stream)))
        return out

    def run_host(self, xs, mode: int, chunked: bool = False, out=None, stream=None):
        """Same op on host slabs: H2D copies, the kernel, D2H copies; returns when done."""
        w, (B, S, H, D), out, ip, op, _ = marshal_slabs(xs, mode, out, "cpu", self.elem_bytes)
        rc = _lib.ulysses_a2a_run_host(self._ctx, ip, op, B, S, H, D, w, mode, int(chunked),
                                       self._stream_handle(stream))
        self._check(rc)
        return out

    def status(self, stream=None) -> None:
        """Synchronise ``stream``; raise if a kernel of this context gave up a wait."""
        self._check(_lib.ulysses_a2a_status(self._ctx, self._stream_handle(stream)))

    def plan(self, xs, mode: int, chunked: bool = False, out=None, knobs=None) -> dict:
        """The path and geometry a run with these tensors would use (host only), with
        this context's forced path and tuning, or the given ``knobs`` dict instead."""
        w, (B, S, H, D), out, ip, op, pitch = marshal_slabs(xs, mode, out, xs[0].device.type,
                                                            self.elem_bytes, allow_pitch=True)
        path, current = self.settings()
        rc, p, msg = _lib.ulysses_a2a_plan_ex(ip, op, B, S, H, D, w, mode,
                                              int(chunked), self.elem_bytes,
                                              row_pitch=pitch, forced_path=path,
                                              **(current if knobs is None else knobs))
        if rc != _lib.OK:
            raise A2AError(rc, msg)
        return p.as_dict()

    def close(self) -> None:
        if self._ctx is not None:
            ctx, self._ctx = self._ctx, None
            rc = _lib.ulysses_a2a_destroy(ctx)
            if rc != _lib.OK:
                raise A2AError(rc, "destroy reported a CUDA error (the handle is released)")

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()
