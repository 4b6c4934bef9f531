"""ctypes binding of libulysses_a2a.so (include/ulysses_a2a.h), same names.

Argument marshalling only: every step of the re-layout runs inside the CUDA
library. If the library is missing this module raises at import; there is no
fallback of any kind.
"""

from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libulysses_a2a.so")

OK = 0
ERR_INVALID = 1
ERR_OVERLAP = 2
ERR_DEVICE = 3
ERR_CUDA = 4
ERR_UNSUPPORTED = 5
ERR_NOMEM = 6
ERR_TIMEOUT = 7
ERR_INTERNAL = 8

PATH_AUTO = 0
PATH_TMA = 1
PATH_VEC = 2
PATH_STAGED = 3

MAX_W = 64
MAX_W_TMA = 8

EXPORTED = (
    "ulysses_a2a_create",
    "ulysses_a2a_destroy",
    "ulysses_a2a_run",
    "ulysses_a2a_run_host",
    "ulysses_a2a_last_error",
    "ulysses_a2a_status",
    "ulysses_a2a_set_path",
    "ulysses_a2a_set_tuning",
    "ulysses_a2a_launch_count",
    "ulysses_a2a_plan",
    "ulysses_a2a_run_noalloc",
    "ulysses_a2a_run_ex",
    "ulysses_a2a_plan_ex",
    "ulysses_a2a_selftest_wait_timeout",
    "ulysses_a2a_get_settings",
    "ulysses_a2a_peer_create",
    "ulysses_a2a_peer_open",
    "ulysses_a2a_peer_publish",
    "ulysses_a2a_peer_pull",
    "ulysses_a2a_peer_pull_packed",
    "ulysses_a2a_peer_window",
    "ulysses_a2a_peer_window_bytes",
    "ulysses_a2a_peer_close",
    "ulysses_a2a_peer_destroy",
)

PEER_HANDLE_BYTES = 128


class PlanT(ctypes.Structure):
    """Mirror of ``ulysses_a2a_plan_t``."""

    _fields_ = [
        ("path", ctypes.c_int32),
        ("vec_bytes", ctypes.c_int32),
        ("row_bytes", ctypes.c_int64),
        ("rows_per_tile", ctypes.c_int64),
        ("tiles_per_block", ctypes.c_int64),
        ("tail_rows", ctypes.c_int64),
        ("units", ctypes.c_int64),
        ("payload_bytes", ctypes.c_int64),
        ("launches", ctypes.c_int32),
        ("grid", ctypes.c_int32),
        ("block", ctypes.c_int32),
        ("stages", ctypes.c_int32),
        ("lookahead", ctypes.c_int32),
        ("producers", ctypes.c_int32),
        ("smem_bytes", ctypes.c_int64),
        ("order", ctypes.c_int32),
        ("chunk_units", ctypes.c_int32),
        ("row_pitch", ctypes.c_int64),
        ("peeled", ctypes.c_int32),
        ("fixed_phase", ctypes.c_int32),
    ]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


class TuningT(ctypes.Structure):
    """Mirror of ``ulysses_a2a_tuning_t`` (speed knobs; defaults keep the library's choice)."""

    _fields_ = [
        ("rows_per_tile", ctypes.c_int32),
        ("ctas_per_sm", ctypes.c_int32),
        ("stages", ctypes.c_int32),
        ("lookahead", ctypes.c_int32),
        ("producers", ctypes.c_int32),
        ("order", ctypes.c_int32),
        ("chunk_units", ctypes.c_int32),
        ("host_chunks", ctypes.c_int32),
        ("staged_form", ctypes.c_int32),
    ]

    DEFAULTS = dict(rows_per_tile=0, ctas_per_sm=0, stages=0, lookahead=0, producers=0,
                    order=-1, chunk_units=-1, host_chunks=0, staged_form=0)

    @classmethod
    def make(cls, **kw):
        vals = dict(cls.DEFAULTS)
        for k, v in kw.items():
            if k not in vals:
                raise TypeError(f"unknown tuning knob {k!r}")
            vals[k] = int(v)
        return cls(**vals)


class DescT(ctypes.Structure):
    """Mirror of ``ulysses_a2a_desc_t``."""

    _fields_ = [
        ("in_slabs", ctypes.POINTER(ctypes.c_void_p)),
        ("out_slabs", ctypes.POINTER(ctypes.c_void_p)),
        ("B", ctypes.c_int64),
        ("S_local", ctypes.c_int64),
        ("H", ctypes.c_int64),
        ("D", ctypes.c_int64),
        ("w", ctypes.c_int32),
        ("mode", ctypes.c_int32),
        ("chunked", ctypes.c_int32),
        ("ntensors", ctypes.c_int32),
        ("row_pitch", ctypes.c_int64),
    ]


def make_desc(in_ptrs, out_ptrs, B, S_local, H, D, w, mode, chunked, row_pitch=0, ntensors=0):
    """A DescT plus the pointer arrays it references (keep both alive together)."""
    ins = ptr_array(in_ptrs) if in_ptrs is not None else None
    outs = ptr_array(out_ptrs) if out_ptrs is not None else None
    d = DescT(ctypes.cast(ins, ctypes.POINTER(ctypes.c_void_p)) if ins is not None else None,
              ctypes.cast(outs, ctypes.POINTER(ctypes.c_void_p)) if outs is not None else None,
              int(B), int(S_local), int(H), int(D), int(w), int(mode), int(chunked),
              int(ntensors), int(row_pitch))
    return d, (ins, outs)


class DescBuffer:
    """One DescT and its two pointer arrays, refilled in place call after call.

    Building a fresh descriptor (structure, arrays, casts) costs several
    microseconds of Python per call, as much as a small launch's kernel. A
    context serves one host thread at a time, so one buffer per context is
    enough; the arrays grow when a call passes more slabs than they hold."""

    def __init__(self, capacity: int = 16):
        self.desc = DescT()
        self.ref = ctypes.byref(self.desc)
        self._cap = 0
        self._grow(capacity)

    def _grow(self, n: int) -> None:
        self.ins = (ctypes.c_void_p * n)()
        self.outs = (ctypes.c_void_p * n)()
        self.desc.in_slabs = ctypes.cast(self.ins, ctypes.POINTER(ctypes.c_void_p))
        self.desc.out_slabs = ctypes.cast(self.outs, ctypes.POINTER(ctypes.c_void_p))
        self._cap = n

    def fill(self, in_ptrs, out_ptrs, B, S_local, H, D, w, mode, chunked, row_pitch=0,
             ntensors=0):
        """Writes one call's arguments; returns the reference to pass to the library."""
        ni, no = len(in_ptrs), len(out_ptrs)
        if ni > self._cap or no > self._cap:
            self._grow(max(ni, no))
        self.ins[:ni] = in_ptrs
        self.outs[:no] = out_ptrs
        d = self.desc
        d.B, d.S_local, d.H, d.D = B, S_local, H, D
        d.w, d.mode, d.chunked, d.ntensors, d.row_pitch = w, mode, chunked, ntensors, row_pitch
        return self.ref


class A2AError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"ulysses_a2a error {code}: {msg}")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is not built; run `python sequence_all_re_b200/build.py` "
            "(the CUDA library is required: there is no fallback path)")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    PP = ctypes.POINTER(ctypes.c_void_p)
    i64 = ctypes.c_int64
    c_int = ctypes.c_int
    lib.ulysses_a2a_create.argtypes = [ctypes.POINTER(P), c_int, c_int]
    lib.ulysses_a2a_create.restype = c_int
    lib.ulysses_a2a_destroy.argtypes = [P]
    lib.ulysses_a2a_destroy.restype = c_int
    run_args = [P, PP, PP, i64, i64, i64, i64, c_int, c_int, c_int, P]
    lib.ulysses_a2a_run.argtypes = run_args
    lib.ulysses_a2a_run.restype = c_int
    lib.ulysses_a2a_run_host.argtypes = run_args
    lib.ulysses_a2a_run_host.restype = c_int
    lib.ulysses_a2a_last_error.argtypes = [P]
    lib.ulysses_a2a_last_error.restype = ctypes.c_char_p
    lib.ulysses_a2a_status.argtypes = [P, P]
    lib.ulysses_a2a_status.restype = c_int
    lib.ulysses_a2a_set_path.argtypes = [P, c_int]
    lib.ulysses_a2a_set_path.restype = c_int
    lib.ulysses_a2a_set_tuning.argtypes = [P, ctypes.POINTER(TuningT)]
    lib.ulysses_a2a_set_tuning.restype = c_int
    lib.ulysses_a2a_launch_count.argtypes = [P]
    lib.ulysses_a2a_launch_count.restype = ctypes.c_uint64
    lib.ulysses_a2a_plan.argtypes = [PP, PP, i64, i64, i64, i64, c_int, c_int, c_int, c_int,
                                     c_int, ctypes.POINTER(TuningT), c_int,
                                     ctypes.POINTER(PlanT), ctypes.c_char_p, ctypes.c_size_t]
    lib.ulysses_a2a_plan.restype = c_int
    lib.ulysses_a2a_run_noalloc.argtypes = [PP, PP, i64, i64, i64, i64, c_int, c_int, c_int, c_int,
                                            P, c_int, ctypes.c_char_p, ctypes.c_size_t]
    lib.ulysses_a2a_run_noalloc.restype = c_int
    lib.ulysses_a2a_run_ex.argtypes = [P, ctypes.POINTER(DescT), P]
    lib.ulysses_a2a_run_ex.restype = c_int
    lib.ulysses_a2a_plan_ex.argtypes = [ctypes.POINTER(DescT), c_int, c_int, ctypes.POINTER(TuningT),
                                        c_int, ctypes.POINTER(PlanT), ctypes.c_char_p,
                                        ctypes.c_size_t]
    lib.ulysses_a2a_plan_ex.restype = c_int
    lib.ulysses_a2a_selftest_wait_timeout.argtypes = [P, ctypes.c_uint32, P]
    lib.ulysses_a2a_selftest_wait_timeout.restype = c_int
    lib.ulysses_a2a_get_settings.argtypes = [P, ctypes.POINTER(ctypes.c_int32),
                                             ctypes.POINTER(TuningT)]
    lib.ulysses_a2a_get_settings.restype = c_int
    lib.ulysses_a2a_peer_create.argtypes = [P, c_int, c_int, ctypes.c_size_t, ctypes.POINTER(P), P]
    lib.ulysses_a2a_peer_create.restype = c_int
    lib.ulysses_a2a_peer_open.argtypes = [P, P]
    lib.ulysses_a2a_peer_open.restype = c_int
    lib.ulysses_a2a_peer_publish.argtypes = [P, P, i64, i64, i64, i64, c_int, i64, ctypes.c_size_t, P]
    lib.ulysses_a2a_peer_publish.restype = c_int
    lib.ulysses_a2a_peer_pull.argtypes = [P, P, i64, i64, i64, i64, c_int, i64, ctypes.c_size_t, P]
    lib.ulysses_a2a_peer_pull.restype = c_int
    lib.ulysses_a2a_peer_pull_packed.argtypes = [P, PP, c_int, i64, i64, i64, i64, c_int,
                                                 ctypes.c_size_t, P]
    lib.ulysses_a2a_peer_pull_packed.restype = c_int
    lib.ulysses_a2a_peer_window.argtypes = [P, c_int]
    lib.ulysses_a2a_peer_window.restype = P
    lib.ulysses_a2a_peer_window_bytes.argtypes = [P]
    lib.ulysses_a2a_peer_window_bytes.restype = ctypes.c_size_t
    lib.ulysses_a2a_peer_close.argtypes = [P]
    lib.ulysses_a2a_peer_close.restype = c_int
    lib.ulysses_a2a_peer_destroy.argtypes = [P]
    lib.ulysses_a2a_peer_destroy.restype = c_int
    return lib


lib = _load()


def ptr_array(ptrs) -> ctypes.Array:
    return (ctypes.c_void_p * len(ptrs))(*[int(p) or None for p in ptrs])


# ---- same-named thin wrappers -------------------------------------------------

def ulysses_a2a_create(device: int, elem_bytes: int) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    rc = lib.ulysses_a2a_create(ctypes.byref(h), int(device), int(elem_bytes))
    if rc != OK:
        raise A2AError(rc, f"create(device={device}, elem_bytes={elem_bytes}) failed")
    return h


def ulysses_a2a_destroy(ctx) -> int:
    return lib.ulysses_a2a_destroy(ctx)


def ulysses_a2a_last_error(ctx) -> str:
    s = lib.ulysses_a2a_last_error(ctx)
    return s.decode() if s else ""


def ulysses_a2a_run(ctx, in_ptrs, out_ptrs, B, S_local, H, D, w, mode, chunked, stream) -> int:
    return lib.ulysses_a2a_run(ctx, ptr_array(in_ptrs), ptr_array(out_ptrs), int(B), int(S_local),
                               int(H), int(D), int(w), int(mode), int(chunked),
                               ctypes.c_void_p(int(stream)))


def ulysses_a2a_run_host(ctx, in_ptrs, out_ptrs, B, S_local, H, D, w, mode, chunked, stream) -> int:
    return lib.ulysses_a2a_run_host(ctx, ptr_array(in_ptrs), ptr_array(out_ptrs), int(B),
                                    int(S_local), int(H), int(D), int(w), int(mode), int(chunked),
                                    ctypes.c_void_p(int(stream)))


def ulysses_a2a_status(ctx, stream) -> int:
    return lib.ulysses_a2a_status(ctx, ctypes.c_void_p(int(stream)))


def ulysses_a2a_set_path(ctx, path: int) -> int:
    return lib.ulysses_a2a_set_path(ctx, int(path))


def ulysses_a2a_set_tuning(ctx, **knobs) -> int:
    """Apply TuningT knobs (rows_per_tile, ctas_per_sm, stages, lookahead, producers,
    order, chunk_units); no knobs restores every default."""
    t = TuningT.make(**knobs)
    return lib.ulysses_a2a_set_tuning(ctx, ctypes.byref(t))


def ulysses_a2a_get_settings(ctx):
    """Returns (rc, forced path, dict of tuning knobs)."""
    path = ctypes.c_int32()
    t = TuningT()
    rc = lib.ulysses_a2a_get_settings(ctx, ctypes.byref(path), ctypes.byref(t))
    return rc, path.value, {name: getattr(t, name) for name, _ in TuningT._fields_}


def ulysses_a2a_launch_count(ctx) -> int:
    return int(lib.ulysses_a2a_launch_count(ctx))


def ulysses_a2a_run_noalloc(in_ptrs, out_ptrs, B, S_local, H, D, w, mode, chunked, elem_bytes,
                            stream, wait=1):
    """The allocation-free entry point (current device). Returns (rc, message)."""
    buf = ctypes.create_string_buffer(256)
    rc = lib.ulysses_a2a_run_noalloc(ptr_array(in_ptrs), ptr_array(out_ptrs), int(B), int(S_local),
                                     int(H), int(D), int(w), int(mode), int(chunked),
                                     int(elem_bytes), ctypes.c_void_p(int(stream)), int(wait),
                                     buf, len(buf))
    return rc, buf.value.decode()


def ulysses_a2a_plan(in_ptrs, out_ptrs, B, S_local, H, D, w, mode, chunked, elem_bytes,
                     forced_path=PATH_AUTO, num_sms=148, **knobs):
    """Host-only planning (no CUDA call). Returns (rc, PlanT, message)."""
    plan = PlanT()
    buf = ctypes.create_string_buffer(256)
    ins = ptr_array(in_ptrs) if in_ptrs is not None else None
    outs = ptr_array(out_ptrs) if out_ptrs is not None else None
    t = TuningT.make(**knobs)
    rc = lib.ulysses_a2a_plan(ins, outs, int(B), int(S_local), int(H), int(D), int(w), int(mode),
                              int(chunked), int(elem_bytes), int(forced_path), ctypes.byref(t),
                              int(num_sms), ctypes.byref(plan), buf, len(buf))
    return rc, plan, buf.value.decode()


def ulysses_a2a_run_ex(ctx, in_ptrs, out_ptrs, B, S_local, H, D, w, mode, chunked, row_pitch,
                       stream, ntensors=0) -> int:
    d, keep = make_desc(in_ptrs, out_ptrs, B, S_local, H, D, w, mode, chunked, row_pitch, ntensors)
    return lib.ulysses_a2a_run_ex(ctx, ctypes.byref(d), ctypes.c_void_p(int(stream)))


def run_ex_ref(ctx, desc_ref, stream) -> int:
    """ulysses_a2a_run_ex on a descriptor already filled (a DescBuffer's ``ref``)."""
    return lib.ulysses_a2a_run_ex(ctx, desc_ref, stream)


def ulysses_a2a_plan_ex(in_ptrs, out_ptrs, B, S_local, H, D, w, mode, chunked, elem_bytes,
                        row_pitch=0, forced_path=PATH_AUTO, num_sms=148, ntensors=0, **knobs):
    """Host-only planning of a descriptor (no CUDA call). Returns (rc, PlanT, message)."""
    d, keep = make_desc(in_ptrs, out_ptrs, B, S_local, H, D, w, mode, chunked, row_pitch,
                        ntensors)
    plan = PlanT()
    buf = ctypes.create_string_buffer(256)
    t = TuningT.make(**knobs)
    rc = lib.ulysses_a2a_plan_ex(ctypes.byref(d), int(elem_bytes), int(forced_path),
                                 ctypes.byref(t), int(num_sms), ctypes.byref(plan), buf, len(buf))
    return rc, plan, buf.value.decode()


# ---- multi-GPU exchange through published windows ------------------------------

def ulysses_a2a_peer_create(ctx, rank: int, world: int, window_bytes: int):
    """Returns (rc, peer handle, the rank's exchange record as bytes)."""
    h = ctypes.c_void_p()
    rec = ctypes.create_string_buffer(PEER_HANDLE_BYTES)
    rc = lib.ulysses_a2a_peer_create(ctx, int(rank), int(world), int(window_bytes),
                                     ctypes.byref(h), rec)
    return rc, h, rec.raw


def ulysses_a2a_peer_open(peer, records) -> int:
    """records: every rank's exchange record (bytes), in rank order."""
    blob = b"".join(bytes(r) for r in records)
    buf = ctypes.create_string_buffer(blob, len(blob))
    return lib.ulysses_a2a_peer_open(peer, buf)


def ulysses_a2a_peer_publish(peer, in_ptr, B, S_local, H, D, mode, row_pitch, stream,
                             window_offset=0) -> int:
    return lib.ulysses_a2a_peer_publish(peer, ctypes.c_void_p(int(in_ptr) or None), int(B),
                                        int(S_local), int(H), int(D), int(mode), int(row_pitch),
                                        int(window_offset), ctypes.c_void_p(int(stream)))


def ulysses_a2a_peer_pull(peer, out_ptr, B, S_local, H, D, mode, row_pitch, stream,
                          window_offset=0) -> int:
    return lib.ulysses_a2a_peer_pull(peer, ctypes.c_void_p(int(out_ptr) or None), int(B),
                                     int(S_local), int(H), int(D), int(mode), int(row_pitch),
                                     int(window_offset), ctypes.c_void_p(int(stream)))


def ulysses_a2a_peer_pull_packed(peer, out_ptrs, ntensors, B, S_local, H, D, mode, stream,
                                 window_offset=0) -> int:
    """One launch for T head-packed tensors: out_ptrs holds T output pointers in
    mode 0, the one packed output in mode 1."""
    return lib.ulysses_a2a_peer_pull_packed(peer, ptr_array(out_ptrs), int(ntensors), int(B),
                                            int(S_local), int(H), int(D), int(mode),
                                            int(window_offset), ctypes.c_void_p(int(stream)))


def ulysses_a2a_peer_window(peer, rank: int) -> int:
    return int(lib.ulysses_a2a_peer_window(peer, int(rank)) or 0)


def ulysses_a2a_peer_window_bytes(peer) -> int:
    return int(lib.ulysses_a2a_peer_window_bytes(peer))


def ulysses_a2a_peer_close(peer) -> int:
    return lib.ulysses_a2a_peer_close(peer)


def ulysses_a2a_peer_destroy(peer) -> int:
    return lib.ulysses_a2a_peer_destroy(peer)
