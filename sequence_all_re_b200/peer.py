"""Multi-GPU Ulysses all-to-all: one process per GPU, exchange through windows.

Each rank holds its own sequence shard ``x_rank`` ([B, S_local, H, D]) on its
own GPU; mode 0 gives every rank ``[B, S_local*w, H//w, D]`` (its head group,
whole sequence), mode 1 undoes it, with the element map of the single-GPU
re-layout (``UlyssesA2A``), of which rank k's part is the output slab k.

The communicator follows the FastVideo API docs' ulysses_a2a helper:

* a device window per rank, built once (``_build``) and reused call after
  call; a call that needs more bytes closes and rebuilds it (window grow in
  ``try_all_to_all_4D``);
* ``chunked=True`` runs the exchange plane by plane on one-plane views
  (``run_armed``);
* the result owns its storage and never aliases the window;
* teardown is collective (``close``): synchronise, agree, release.

One exchange (per call, or per plane when chunked), as in the pypto-lib pull
request "pipeline HCA AllToAll into O-A", which publishes into a distributed
window and has consumers load from it after a handshake:
publish (own input into one half of own window) -> barrier -> pull (one
kernel reads this rank's share out of that half of every window over NVLink
and writes the local output). Exchanges use the two halves of the windows in
turn, so a publish needs no barrier of its own: the half it overwrites was
last read two exchanges back, and the previous exchange's barrier completed
on every rank after that rank's pull from it (each rank's exchanges are
ordered on one stream). With ``input_buffer()`` the producer of the slab
writes it into the next half itself (that pull request's publishing workers),
and the publish copy drops out. The barrier is a collective of the process
group on the caller's stream (NCCL: a one-element all-reduce, stream ordered,
no host wait) or, for host-only backends such as gloo, a stream synchronise
plus a group barrier. No kernel waits for another GPU.

Every copy runs in ``libulysses_a2a.so`` (``ulysses_a2a_peer_*``); this module
only sequences the calls and the group's collectives.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import UlyssesA2A, _lib, mode0_local_tuple, output_shape
from . import row_pitch as slab_row_pitch
from ._lib import A2AError

__all__ = ["PeerExchange", "NativePeer"]


class _DeviceBytes:
    """n bytes of device memory at ptr, exposed through the CUDA array interface
    (so torch can view the window without copying it)."""

    def __init__(self, ptr: int, n: int):
        self.__cuda_array_interface__ = {"data": (int(ptr), False), "shape": (int(n),),
                                         "typestr": "|u1", "version": 2, "strides": None}


class NativePeer:
    """The C ABI's peer object for one rank (marshalling only)."""

    def __init__(self, device, elem_bytes: int):
        self.a2a = UlyssesA2A(device, elem_bytes)
        self.device = self.a2a.device
        self.elem_bytes = self.a2a.elem_bytes
        self._peer = None

    def _check(self, rc):
        if rc != _lib.OK:
            raise A2AError(rc, self.a2a.last_error())

    def create(self, rank: int, world: int, nbytes: int) -> bytes:
        if self._peer is not None:
            raise RuntimeError("window already built")
        rc, h, rec = _lib.ulysses_a2a_peer_create(self.a2a._ctx, rank, world, nbytes)
        self._check(rc)
        self._peer = h
        self._rank = rank
        self._nbytes = int(nbytes)
        return rec

    def open(self, records) -> None:
        self._check(_lib.ulysses_a2a_peer_open(self._peer, records))

    def publish(self, x, B, S, H, D, mode, row_pitch, stream, window_offset=0) -> None:
        self._check(_lib.ulysses_a2a_peer_publish(self._peer, x.data_ptr(), B, S, H, D, mode,
                                                  row_pitch, stream.cuda_stream, window_offset))

    def pull(self, out, B, S, H, D, mode, row_pitch, stream, window_offset=0) -> None:
        self._check(_lib.ulysses_a2a_peer_pull(self._peer, out.data_ptr(), B, S, H, D, mode,
                                               row_pitch, stream.cuda_stream, window_offset))

    def pull_packed(self, outs, T, B, S, H, D, mode, stream, window_offset=0) -> None:
        """One launch for T head-packed tensors: ``outs`` is T tensors (mode 0)
        or the one packed [B, S, T, H, D] output (mode 1)."""
        ptrs = [t.data_ptr() for t in outs] if mode == 0 else [outs.data_ptr()]
        self._check(_lib.ulysses_a2a_peer_pull_packed(self._peer, ptrs, T, B, S, H, D, mode,
                                                      stream.cuda_stream, window_offset))

    def window(self, rank: int) -> int:
        return _lib.ulysses_a2a_peer_window(self._peer, rank) if self._peer is not None else 0

    def window_tensor(self, shape, dtype, offset: int = 0) -> torch.Tensor:
        """This rank's window from byte ``offset`` on as a dense tensor (no copy;
        valid until the window is released)."""
        n = torch.empty((), dtype=dtype).element_size()
        for v in shape:
            n *= int(v)
        if self._peer is None or offset + n > self._nbytes:
            raise ValueError("the window is not built or is smaller than the tensor")
        raw = torch.as_tensor(_DeviceBytes(self.window(self._rank) + offset, n),
                              device=self.device)
        return raw.view(dtype).view(tuple(shape))

    def unmap(self) -> None:
        if self._peer is not None:
            self._check(_lib.ulysses_a2a_peer_close(self._peer))

    def release(self) -> None:
        if self._peer is not None:
            h, self._peer = self._peer, None
            rc = _lib.ulysses_a2a_peer_destroy(h)
            if rc != _lib.OK:
                raise A2AError(rc, "peer_destroy reported a CUDA error (the handle is released)")

    def abandon(self) -> None:
        """Forget the peer object without unmapping or freeing its window: the
        memory stays allocated until the process exits (for a teardown the
        ranks could not agree on)."""
        self._peer = None

    @property
    def launch_count(self) -> int:
        return self.a2a.launch_count

    def current_stream(self):
        return torch.cuda.current_stream(self.device)

    def synchronize(self) -> None:
        torch.cuda.synchronize(self.device)

    def close(self) -> None:
        self.release()
        self.a2a.close()


class PeerExchange:
    """This rank's side of the multi-GPU Ulysses all-to-all over ``group``."""

    def __init__(self, group=None, device=None, elem_bytes: int = 2, barrier: str = "auto",
                 native=None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        if native is None:
            native = NativePeer(torch.cuda.current_device() if device is None else device,
                                elem_bytes)
        self.native = native
        self.device = self.native.device
        self.elem_bytes = int(elem_bytes)
        if barrier == "auto":
            barrier = "stream" if dist.get_backend(group) == "nccl" else "host"
        if barrier not in ("stream", "host"):
            raise ValueError("barrier must be 'auto', 'stream' or 'host'")
        self.barrier_kind = barrier
        self._flag = (torch.zeros(1, dtype=torch.int32, device=self.device)
                      if barrier == "stream" else None)
        self._nbytes = 0               # each rank's window: two halves of _nbytes // 2
        self._half = 0                 # the half the next exchange publishes into
        self._armed = False
        self._agreed = set()           # call signatures every rank has confirmed
        self._in_place = None          # (address, offset) handed out by input_buffer()
        self.disabled_reason = None

    # ---------------------------------------------------------- group helpers
    def _gather(self, obj):
        out = [None] * self.world
        dist.all_gather_object(out, obj, group=self.group)
        return out

    def _agree(self, ok: bool) -> bool:
        return all(self._gather(bool(ok)))

    def _barrier(self, stream) -> None:
        if self.barrier_kind == "stream":
            with torch.cuda.stream(stream):
                dist.all_reduce(self._flag, group=self.group)
        else:
            stream.synchronize()
            dist.barrier(group=self.group)

    def _disable(self, reason: str) -> None:
        self.disabled_reason = reason

    # --------------------------------------------------------------- lifecycle
    def build(self, nbytes: int) -> bool:
        """Collectively allocate every rank's window (``nbytes`` each) and map
        the peers' windows. Returns whether every rank succeeded."""
        rec, ok = None, True
        try:
            rec = self.native.create(self.rank, self.world, int(nbytes))
        except (A2AError, RuntimeError):
            ok = False
        recs = self._gather(rec if ok else None)
        if any(r is None for r in recs):
            self._release_after_failure()
            return False
        try:
            self.native.open(recs)
        except A2AError:
            ok = False
        if not self._agree(ok):
            # every rank unmaps and waits for the others before freeing
            self._teardown_mapped()
            return False
        self._nbytes = int(nbytes)
        self._armed = True
        return True

    def _release_after_failure(self) -> None:
        try:
            self.native.release()
        except A2AError:
            pass
        self._nbytes = 0
        self._armed = False

    def _teardown_mapped(self) -> bool:
        ok = True
        try:
            self.native.unmap()
        except A2AError:
            ok = False
        dist.barrier(group=self.group)          # no peer maps our window any more
        try:
            self.native.release()
        except A2AError:
            ok = False
        self._nbytes = 0
        self._armed = False
        return ok

    def close(self) -> bool:
        """Collective teardown of the windows; returns whether every rank completed it."""
        all_armed = self._agree(self._armed)
        all_unarmed = self._agree(not self._armed)
        if all_unarmed:
            return True
        if not all_armed:
            # An armed/unarmed split cannot be torn down safely: a peer may still
            # map this window. Leave it allocated until the process exits, as the
            # FastVideo communicator does, and disable the exchange.
            self.native.abandon()
            self._nbytes = 0
            self._armed = False
            self._disable("ranks disagreed on whether a window was built during teardown")
            return False
        sync_ok = True
        try:
            self.native.synchronize()
        except RuntimeError:
            sync_ok = False
        if not self._agree(sync_ok):
            self._disable("a peer rank could not synchronize before window teardown")
            return False
        return self._agree(self._teardown_mapped())

    def shutdown(self) -> None:
        """close() and release the library context (collective)."""
        self.close()
        self.native.close()

    # -------------------------------------------------------------------- the op
    def _agree_signature(self, sig) -> None:
        if sig not in self._agreed:
            sigs = self._gather(sig)
            if any(s != sig for s in sigs):
                raise ValueError(f"ranks called the exchange with different arguments: {sigs}")
            self._agreed.add(sig)

    def _ensure_window(self, need: int) -> None:
        """Windows whose two halves hold at least ``need`` bytes each (256-byte
        aligned halves)."""
        span = (need + 255) // 256 * 256
        if 2 * span > self._nbytes:
            if self._armed and not self.close():
                raise RuntimeError("window teardown before growing failed")
            if not self.build(2 * span):
                self._disable("a rank could not build its window")
                raise RuntimeError("peer exchange: window build failed on some rank")
            self._half = 0
            self._in_place = None

    def _take_half(self) -> int:
        """Byte offset of the window half this exchange publishes into and pulls
        from; the next exchange takes the other half. A half that
        input_buffer() handed out and no exchange used is taken again (it was
        never read, and taking the other one would overwrite the half the last
        exchange's pulls may still read)."""
        if self._in_place is not None:
            self._in_place = None
            self._half ^= 1
        off = self._half * (self._nbytes // 2)
        self._half ^= 1
        return off

    def input_buffer(self, shape, dtype=torch.bfloat16, stream=None) -> torch.Tensor:
        """This rank's window as a dense tensor of ``shape``, for an in-place input.

        Collective: every rank calls it with the same shape. It hands out the
        window half the next exchange uses, which no rank reads any more once
        the previous exchange's barrier has passed on this rank's stream, so
        the caller may write its slab straight into the returned tensor on
        that stream (for example as the output of the projection that produces
        it) and then pass that tensor to ``all_to_all_4d`` with
        ``chunked=False``, which skips the publish copy. The tensor is valid
        until the window is rebuilt or closed.
        """
        if self.disabled_reason is not None:
            raise RuntimeError(f"peer exchange disabled: {self.disabled_reason}")
        shape = tuple(int(v) for v in shape)
        if len(shape) != 4 or torch.empty((), dtype=dtype).element_size() != self.elem_bytes:
            raise ValueError(f"a 4D shape of {self.elem_bytes}-byte elements is required")
        need = self.elem_bytes
        for v in shape:
            need *= v
        self._agree_signature(("input_buffer", shape, dtype))
        self._ensure_window(need)
        off = self._take_half()
        t = self.native.window_tensor(shape, dtype, off)
        self._in_place = (t.data_ptr(), off)
        return t

    def all_to_all_4d_packed(self, x, mode: int, out=None, stream=None):
        """Exchange T tensors packed along the head dimension with one barrier.

        mode 0: ``x`` is this rank's contiguous [B, S_local, T, H, D] slab (for
        example its packed q/k/v projection output); returns T tensors
        [B, S_local*w, H//w, D]. It is published whole, and each tensor is
        pulled from the windows at its head offset with row pitch T*H*D.
        mode 1: ``x`` is a list of T tensors [B, S_local*w, H//w, D]; returns
        the packed [B, S_local, T, H, D] slab (``out`` may be given). The T
        slabs share the window at consecutive offsets, and each is pulled
        into its slot of the packed output.
        Same bytes as T calls of ``all_to_all_4d``; one barrier instead of T,
        and one pull launch for all T tensors.
        """
        if self.disabled_reason is not None:
            raise RuntimeError(f"peer exchange disabled: {self.disabled_reason}")
        if mode not in (0, 1):
            raise ValueError("mode must be 0 or 1")
        w, E = self.world, self.elem_bytes
        if mode == 0:
            if x.dim() != 5 or not x.is_contiguous():
                raise ValueError("mode 0 takes a contiguous [B, S_local, T, H, D] slab")
            B, S, T, H, D = (int(v) for v in x.shape)
            srcs = [x]
            dtype, device = x.dtype, x.device
        else:
            T = len(x)
            if T < 1 or x[0].dim() != 4:
                raise ValueError("mode 1 takes a list of T tensors [B, S_local*w, H/w, D]")
            B, Sg, Hw, D = (int(v) for v in x[0].shape)
            S, H = Sg // w, Hw * w
            srcs = list(x)
            dtype, device = x[0].dtype, x[0].device
            if Sg % w or any(tuple(t.shape) != (B, Sg, Hw, D) or not t.is_contiguous()
                             for t in srcs):
                raise ValueError("the T tensors must be contiguous [B, S_local*w, H/w, D]")
        if H % w:
            raise ValueError("H must be divisible by the world size")
        if any(t.device != self.device or t.element_size() != E for t in srcs):
            raise ValueError(f"tensors must hold {E}-byte elements on {self.device}")
        slab = B * S * H * D * E                     # one tensor's slab, either layout
        if mode == 0:
            outs = out if out is not None else [
                torch.empty((B, S * w, H // w, D), dtype=dtype, device=device) for _ in range(T)]
        else:
            outs = out if out is not None else torch.empty((B, S, T, H, D), dtype=dtype,
                                                           device=device)
        if slab == 0:
            return outs
        self._agree_signature(("packed", mode, T, B, S, H, D, dtype))
        if mode == 1 and not outs.is_contiguous():
            raise ValueError("the packed output must be contiguous")
        self._ensure_window(T * slab)
        if stream is None:
            stream = self.native.current_stream()
        off = self._take_half()
        if mode == 0:
            # the packed rows published whole: T*H heads of D
            self.native.publish(x, B, S, T * H, D, 0, 0, stream, window_offset=off)
        else:
            for t in range(T):
                self.native.publish(srcs[t], B, S, H, D, 1, 0, stream,
                                    window_offset=off + t * slab)
        self._barrier(stream)        # every window holds its slabs
        self.native.pull_packed(outs, T, B, S, H, D, mode, stream, window_offset=off)
        return outs

    def all_to_all_4d(self, x: torch.Tensor, mode: int, chunked: bool = False, out=None,
                      stream=None) -> torch.Tensor:
        """Exchange this rank's slab ``x``; returns this rank's output slab.

        mode 0: ``x`` is [B, S_local, H, D] (contiguous, or a row-pitched view
        such as q of a packed [B, S, 3, H, D] buffer) -> [B, S_local*w, H//w, D].
        mode 1: ``x`` is [B, S_local*w, H//w, D] -> [B, S_local, H, D] (``out``
        may be a row-pitched view). Every rank calls it with the same shape,
        mode and chunking.
        """
        if self.disabled_reason is not None:
            raise RuntimeError(f"peer exchange disabled: {self.disabled_reason}")
        if mode not in (0, 1):
            raise ValueError("mode must be 0 or 1")
        if x.dim() != 4 or x.device != self.device or x.element_size() != self.elem_bytes:
            raise ValueError(f"x must be a 4D tensor of {self.elem_bytes}-byte elements on "
                             f"{self.device}")
        w = self.world
        if (mode == 0 and x.shape[2] % w) or (mode == 1 and x.shape[1] % w):
            raise ValueError("H (mode 0) or S_global (mode 1) must be divisible by the world size")
        B, S, H, D = mode0_local_tuple(tuple(x.shape), mode, w)
        oshape = output_shape(tuple(x.shape), mode, w)
        if out is None:
            out = torch.empty(oshape, dtype=x.dtype, device=x.device)
        elif tuple(out.shape) != oshape or out.dtype != x.dtype or out.device != x.device:
            raise ValueError(f"out must be {oshape} {x.dtype} on {x.device}")
        strided, dense = (x, out) if mode == 0 else (out, x)
        pitch = slab_row_pitch([strided], allow_pitch=True)
        if not dense.is_contiguous():
            raise ValueError("the [B, S_local*w, H/w, D] slab must be contiguous")
        if B * S * H * D == 0:
            return out
        planes = B if chunked else 1
        need = (1 if chunked else B) * S * H * D * self.elem_bytes
        own = self.native.window(self.rank) if self._armed else 0
        in_place = own != 0 and own <= x.data_ptr() < own + self._nbytes
        self._agree_signature((mode, bool(chunked), B, S, H, D, x.dtype, in_place))
        if stream is None:
            stream = self.native.current_stream()
        if in_place:
            # the slab was written into the half input_buffer() handed out
            if (chunked or not x.is_contiguous() or self._in_place is None
                    or self._in_place[0] != x.data_ptr()):
                raise ValueError("an input in the window must come from input_buffer() and be "
                                 "exchanged whole (chunked=False)")
            off = self._in_place[1]
            self._in_place = None
            self._barrier(stream)    # every window holds its slab
            self.native.pull(out, B, S, H, D, mode, pitch if mode == 1 else 0, stream,
                             window_offset=off)
            return out
        self._ensure_window(need)
        nb = 1 if chunked else B
        for b in range(planes):
            xv = x[b:b + 1] if chunked else x
            ov = out[b:b + 1] if chunked else out
            off = self._take_half()
            self.native.publish(xv, nb, S, H, D, mode, pitch if mode == 0 else 0, stream,
                                window_offset=off)
            self._barrier(stream)    # every window holds this plane
            self.native.pull(ov, nb, S, H, D, mode, pitch if mode == 1 else 0, stream,
                             window_offset=off)
        return out
