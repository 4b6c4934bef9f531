"""CPU oracle for the Ulysses 4D all-to-all re-layout (TEST INFRASTRUCTURE).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package. The product path (``sequence_all_re_b200``) never
imports, loads or calls it, and the two share no code.

The arithmetic lives in ``ulysses_oracle.c`` (plain per-element nested loops,
built with gcc into ``libulysses_oracle.so`` next to it). This wrapper only
derives output shapes the way the FastVideo API docs' ``run_armed`` does and
hands raw CPU buffers to the C loops:

  * mode 0: input ``[B, S_local, H, D]`` per rank -> output
    ``[B, S_local*w, H//w, D]``;
  * mode 1: input ``[B, S_global, H_local, D]`` per rank, with
    ``S_local = S_global // w`` and ``H = H_local * w`` -> output
    ``[B, S_local, H, D]``.

Parity status: every function here is pinned (see tests/test_oracle_pins.py and
tests/test_oracle_mutations.py); none is "parity unpinned".
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ulysses_oracle.c")
_LIB = os.path.join(_HERE, "libulysses_oracle.so")
_LIB_OMP = os.path.join(_HERE, "libulysses_oracle_omp.so")
_lib = None
_lib_omp = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB, extra=()) -> str:
    """Compile the oracle's C source with gcc into a shared library."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-Wall", "-Werror",
               *extra, "-o", out, src]
        subprocess.run(cmd, check=True)
    return out


def build_omp(force: bool = False) -> str:
    """The same source built with OpenMP: the outer (r, b) loops run on every
    host core (same results, element order of the copies aside)."""
    return build(force, _SRC, _LIB_OMP, extra=("-fopenmp",))


def omp_lib() -> ctypes.CDLL:
    """The OpenMP build, loaded once."""
    global _lib_omp
    if _lib_omp is None:
        _lib_omp = load_library(build_omp())
    return _lib_omp


def omp_threads() -> int:
    """Threads the OpenMP build uses (OMP_NUM_THREADS, else the cores this
    process may run on)."""
    v = os.environ.get("OMP_NUM_THREADS", "").split(",")[0].strip()
    if v.isdigit() and int(v) > 0:
        return int(v)
    return len(os.sched_getaffinity(0))


def load_library(path: str) -> ctypes.CDLL:
    lib = ctypes.CDLL(path)
    for name in ("oracle_ulysses_a2a", "oracle_ulysses_a2a_chunked"):
        fn = getattr(lib, name)
        fn.restype = ctypes.c_int
        fn.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_void_p),
                       ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                       ctypes.c_int, ctypes.c_int, ctypes.c_int]
    fn = lib.oracle_ulysses_a2a_pitched
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_void_p),
                   ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                   ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64]
    return lib


def _get_lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = load_library(build())
    return _lib


def output_shape(in_shape, mode: int, w: int) -> tuple:
    """Output slab shape from an input slab shape, as ``run_armed`` derives it."""
    if mode == 0:
        B, S_local, H, D = in_shape
        return (B, S_local * w, H // w, D)
    B, S_global, H_local, D = in_shape
    S_local, H = S_global // w, H_local * w
    return (B, S_local, H, D)


def mode0_local_tuple(in_shape, mode: int, w: int) -> tuple:
    """(B, S_local, H, D) as the native op receives it in either mode."""
    if mode == 0:
        return tuple(int(v) for v in in_shape)
    B, S_global, H_local, D = in_shape
    return (int(B), int(S_global) // w, int(H_local) * w, int(D))


def ulysses_a2a(inputs, mode: int, chunked: bool = False, lib: ctypes.CDLL | None = None):
    """Run the re-layout on CPU tensors ``inputs`` (one per rank, same shape/dtype).

    Returns a list of ``w`` new CPU tensors. Every output byte is pre-filled with
    0xFF, so an element the loops never write stays visibly wrong.
    """
    lib = lib or _get_lib()
    w = len(inputs)
    if w < 1:
        raise ValueError("need at least one rank slab")
    shape = tuple(inputs[0].shape)
    dt = inputs[0].dtype
    for t in inputs:
        if tuple(t.shape) != shape or t.dtype != dt or t.device.type != "cpu":
            raise ValueError("rank slabs must share shape and dtype and live on the CPU")
    if len(shape) != 4:
        raise ValueError("rank slabs are 4D")
    if mode == 0 and shape[2] % w != 0:
        raise ValueError("H must be divisible by w")
    if mode == 1 and shape[1] % w != 0:
        raise ValueError("S_global must be divisible by w")
    B, S_local, H, D = mode0_local_tuple(shape, mode, w)
    out_shape = output_shape(shape, mode, w)
    ins = [t.contiguous() for t in inputs]
    outs = []
    for _ in range(w):
        o = torch.empty(out_shape, dtype=dt)
        o.view(torch.uint8).fill_(0xFF) if o.numel() else None
        outs.append(o)
    in_arr = (ctypes.c_void_p * w)(*[t.data_ptr() or None for t in ins])
    out_arr = (ctypes.c_void_p * w)(*[t.data_ptr() or None for t in outs])
    fn = lib.oracle_ulysses_a2a_chunked if chunked else lib.oracle_ulysses_a2a
    rc = fn(in_arr, out_arr, B, S_local, H, D, w, int(mode), ins[0].element_size())
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (rc={rc})")
    return outs


def ulysses_a2a_pitched(bufs, mode: int, w: int, B: int, S_local: int, H: int, D: int,
                        row_pitch: int, offset: int = 0, out_bufs=None,
                        lib: ctypes.CDLL | None = None):
    """The re-layout with a row pitch on the [B, S_local, H, D] side.

    ``bufs``: w 1-D CPU tensors (any dtype) holding the input slabs; in mode 0
    each is a pitched buffer read from element ``offset`` on (for example a
    packed QKV projection output, offset selecting q, k or v), in mode 1 each is
    a dense [B, S_local*w, H//w, D] slab. ``out_bufs``: w 1-D CPU tensors
    receiving the output (mode 0: dense; mode 1: pitched, written from
    ``offset`` on, gap elements untouched); allocated and 0xFF-filled if None.
    Returns the output buffers.
    """
    lib = lib or _get_lib()
    dt = bufs[0].dtype
    E = bufs[0].element_size()
    if out_bufs is None:
        n = (B * S_local * H * D) if mode == 0 else ((B * S_local - 1) * row_pitch + H * D + offset)
        out_bufs = []
        for _ in range(w):
            o = torch.empty(n, dtype=dt)
            o.view(torch.uint8).fill_(0xFF)
            out_bufs.append(o)
    in_off = offset if mode == 0 else 0
    out_off = offset if mode == 1 else 0
    in_arr = (ctypes.c_void_p * w)(*[t.data_ptr() + in_off * E for t in bufs])
    out_arr = (ctypes.c_void_p * w)(*[t.data_ptr() + out_off * E for t in out_bufs])
    rc = lib.oracle_ulysses_a2a_pitched(in_arr, out_arr, B, S_local, H, D, w, int(mode), E,
                                        int(row_pitch))
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (rc={rc})")
    return out_bufs
