"""The C-ABI library without a GPU: it loads, exports what the header declares,
and its host-only planner validates arguments and lays out work correctly."""

import ctypes
import os
import re

import pytest

from sequence_all_re_b200 import _lib
from sequence_all_re_b200._lib import (ERR_INVALID, ERR_OVERLAP, ERR_UNSUPPORTED, OK, PATH_AUTO,
                                       PATH_STAGED, PATH_TMA, PATH_VEC, ulysses_a2a_plan)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ulysses_a2a.h")

MiB = 1 << 20


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ulysses_a2a_\w+)\s*\(", text)))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    for n in ("ulysses_a2a_create", "ulysses_a2a_destroy", "ulysses_a2a_run"):
        assert n in names
    assert sorted(names) == sorted(_lib.EXPORTED)


def test_header_constants_match_the_binding():
    text = open(HEADER).read()
    defines = {m.group(1): int(m.group(2))
               for m in re.finditer(r"#define\s+ULYSSES_A2A_(\w+)\s+(\d+)", text)}
    binding = {"OK": _lib.OK, "ERR_INVALID": _lib.ERR_INVALID, "ERR_OVERLAP": _lib.ERR_OVERLAP,
               "ERR_DEVICE": _lib.ERR_DEVICE, "ERR_CUDA": _lib.ERR_CUDA,
               "ERR_UNSUPPORTED": _lib.ERR_UNSUPPORTED, "ERR_NOMEM": _lib.ERR_NOMEM,
               "ERR_TIMEOUT": _lib.ERR_TIMEOUT, "ERR_INTERNAL": _lib.ERR_INTERNAL,
               "PATH_AUTO": _lib.PATH_AUTO, "PATH_TMA": _lib.PATH_TMA, "PATH_VEC": _lib.PATH_VEC,
               "PATH_STAGED": _lib.PATH_STAGED,
               "MAX_W": _lib.MAX_W, "MAX_W_TMA": _lib.MAX_W_TMA,
               "PEER_HANDLE_BYTES": _lib.PEER_HANDLE_BYTES}
    for name, value in binding.items():
        assert defines[name] == value, name
    # every status code the header defines is mirrored
    assert {k for k in defines if k == "OK" or k.startswith("ERR_")} <= set(binding)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(_lib.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_plan_struct_layout_matches_header():
    # int32 path, vec_bytes; 6 x int64; 6 x int32; int64; 2 x int32; int64;
    # 2 x int32 (peeled, fixed_phase) -> 112 bytes
    assert ctypes.sizeof(_lib.PlanT) == 112
    # two pointers, 4 x int64, 4 x int32, int64 -> 72 bytes
    assert ctypes.sizeof(_lib.DescT) == 72


def fake_slabs(w, slab_bytes, base=1 << 40, align=256, gap=0):
    """Distinct, non-overlapping fake addresses (never dereferenced)."""
    step = (slab_bytes + gap + align - 1) // align * align
    ins = [base + k * step for k in range(w)]
    outs = [base + (w + k) * step for k in range(w)]
    return ins, outs


def plan(w, B, S, H, D, mode=0, chunked=0, E=2, **kw):
    ins, outs = fake_slabs(w, B * S * H * D * E)
    return ulysses_a2a_plan(ins, outs, B, S, H, D, w, mode, chunked, E, **kw)


# ---- geometry at the benchmark configurations -------------------------------

def test_plan_default_workload_tma():
    rc, p, msg = plan(4, 1, 8192, 24, 128)
    assert rc == OK, msg
    assert p.path == PATH_TMA
    assert p.row_bytes == 6 * 128 * 2
    assert p.rows_per_tile == 8 * 1024 // 1536        # 5 rows, ~8 KB tiles
    assert p.tiles_per_block == -(-8192 // 5)
    assert p.tail_rows == 8192 % 5 == 2
    assert p.units == 4 * 1 * 4 * p.tiles_per_block
    assert p.payload_bytes == 192 * MiB
    assert p.launches == 1
    # default schedule: one short-lived single-warp CTA per 7.5 KB tile, at most
    # round(100 KB / 7.5 KB) = 13 resident per SM: 228 KB / 13 - 1 KB reserved,
    # rounded down to 1 KB = 16 KB of shared memory each
    assert p.producers == 1 and p.block == 32 and p.stages == 1 and p.lookahead == 1
    assert p.chunk_units == 1 and p.grid == p.units == 26224
    assert p.smem_bytes == 16 * 1024
    assert (228 * 1024) // (p.smem_bytes + 1024) == 13
    assert p.order == 1
    # the residency cap is the ctas_per_sm knob: 12 CTAs -> 18 KB each
    rc, q, _ = plan(4, 1, 8192, 24, 128, ctas_per_sm=12)
    assert rc == OK and q.smem_bytes == 18 * 1024 and (228 * 1024) // (q.smem_bytes + 1024) == 12
    # four producers per CTA: the cap drops to round(100 / 30) = 3 CTAs per SM
    rc, q, _ = plan(4, 1, 8192, 24, 128, producers=4, chunk_units=4)
    assert rc == OK and q.block == 128 and q.grid == -(-q.units // 4)
    assert q.smem_bytes == (228 * 1024 // 3 - 1024) // 1024 * 1024
    # the persistent schedule: one CTA per SM, 4 producers x 4-stage rings
    rc, q, _ = plan(4, 1, 8192, 24, 128, chunk_units=0)
    assert rc == OK and q.chunk_units == 0 and q.grid == 148
    assert (q.producers, q.stages, q.lookahead, q.smem_bytes) == (4, 16, 2, 16 * 8 * 1024)


def test_plan_ragged_tail_rows():
    rc, p, _ = plan(8, 2, 4725, 40, 128)
    assert rc == OK and p.path == PATH_TMA
    assert p.row_bytes == 5 * 128 * 2
    assert p.rows_per_tile == 6 and p.tail_rows == 3           # 4725 = 787 * 6 + 3
    rc, p, _ = plan(8, 2, 4725, 40, 128, rows_per_tile=32)
    assert rc == OK
    assert p.rows_per_tile == 32 and p.tail_rows == 4725 - 147 * 32 == 21
    assert p.tiles_per_block == 148
    assert p.units == 8 * 2 * 8 * 148
    # a 64-row tile would be 80 KB: the TMA path caps tiles at 64 KB (51 rows)
    rc, p, _ = plan(8, 2, 4725, 40, 128, rows_per_tile=64)
    assert rc == OK and p.rows_per_tile == 51 and p.tail_rows == 4725 % 51
    rc, p, _ = plan(8, 2, 4725, 40, 128, rows_per_tile=64, forced_path=PATH_VEC)
    assert rc == OK and p.rows_per_tile == 64 and p.tail_rows == 53


def test_plan_four_planes_chunked_launches():
    rc, p, _ = plan(4, 4, 16384, 32, 64, chunked=1)
    assert rc == OK and p.path == PATH_TMA
    assert p.launches == 4
    assert p.units == 4 * 1 * 4 * p.tiles_per_block     # one plane per launch
    rc, q, _ = plan(4, 4, 16384, 32, 64, chunked=0)
    assert q.launches == 1 and q.units == 4 * p.units
    assert p.payload_bytes == q.payload_bytes == 1 << 30


def test_plan_windowed_chunked_variant():
    rc, p, _ = plan(4, 4, 16384, 32, 64, chunked=2)
    assert rc == OK and p.launches == 4
    rc, q, _ = plan(4, 4, 16384, 32, 64, chunked=1)
    assert p.units == q.units


def test_plan_tiny_workload():
    # 64 KiB: AUTO takes the vector kernel (lower latency below 64 MiB), with
    # the smallest units (2 KB: 8 rows of 256 B) so that every SM gets work
    rc, p, _ = plan(2, 1, 64, 4, 64)
    assert rc == OK and p.path == PATH_VEC and p.vec_bytes == 16
    assert p.rows_per_tile == 8 and p.tail_rows == 0 and p.tiles_per_block == 8
    assert p.units == 2 * 2 * 8 and p.grid == p.units
    # forced onto TMA: one-tile CTAs of 32 rows
    rc, p, _ = plan(2, 1, 64, 4, 64, forced_path=PATH_TMA)
    assert rc == OK and p.path == PATH_TMA
    assert p.rows_per_tile == 32 and p.tail_rows == 0 and p.tiles_per_block == 2
    assert p.units == 8 and p.chunk_units == 1 and p.grid == 8


def test_auto_switches_to_tma_above_64_mib_per_launch():
    # w=4, H=16, D=128 bf16: 16 KB per sequence row of all ranks
    rc, p, _ = plan(4, 1, 4096, 16, 128)                # 64 MiB: vector kernel
    assert rc == OK and p.path == PATH_VEC and p.payload_bytes == 64 << 20
    assert p.rows_per_tile == 12 * 1024 // (4 * 128 * 2)   # 12 KB units again
    rc, p, _ = plan(4, 1, 4097, 16, 128)                # just above: TMA
    assert rc == OK and p.path == PATH_TMA
    # chunked: the launch is one plane
    rc, p, _ = plan(4, 2, 4096, 16, 128)                # 128 MiB in one launch: TMA
    assert rc == OK and p.path == PATH_TMA
    rc, p, _ = plan(4, 2, 4096, 16, 128, chunked=1)     # 64 MiB per launch: vector
    assert rc == OK and p.path == PATH_VEC


def test_rows_never_exceed_sequence():
    rc, p, _ = plan(2, 1, 3, 2, 8)
    assert rc == OK and p.rows_per_tile == 3 and p.tiles_per_block == 1


# ---- path selection --------------------------------------------------------

def test_runs_off_16_bytes_take_the_staged_path():
    # AUTO re-aligns in shared memory (16-byte global accesses, pieces of the
    # width the run allows); the vector path, when forced, uses that width
    rc, p, _ = plan(2, 1, 16, 4, 3)             # D*E = 6 bytes
    assert rc == OK and p.path == PATH_STAGED and p.vec_bytes == 4   # run = 2*3*2 = 12 B
    rc, p, _ = plan(2, 1, 16, 4, 3, forced_path=PATH_VEC)
    assert rc == OK and p.path == PATH_VEC and p.vec_bytes == 4
    rc, p, _ = plan(2, 1, 16, 2, 5, E=1)        # run = 5 B
    assert rc == OK and p.path == PATH_STAGED and p.vec_bytes == 1
    rc, p, _ = plan(2, 1, 16, 2, 5, E=1, forced_path=PATH_VEC)
    assert rc == OK and p.path == PATH_VEC and p.vec_bytes == 1


def test_staged_geometry():
    # 200-byte runs, 8 head groups of 1600-byte rows: one unit per (b, j, tile)
    # covering every head group
    # (8-byte vectors: AUTO keeps the vector path, so the staged path is forced)
    # AUTO: the fixed-phase form (8-byte pieces), both modes
    for mode in (0, 1):
        rc, p, _ = plan(8, 2, 4725, 8, 100, mode=mode)
        assert rc == OK and p.path == PATH_STAGED and p.vec_bytes == 8 and p.fixed_phase == 1
    # dense and aligned alike, the fixed-phase form: units of 32 KB (20 rows)
    rc, p, _ = plan(8, 2, 4725, 8, 100, forced_path=PATH_STAGED)
    assert rc == OK and p.path == PATH_STAGED and p.vec_bytes == 8 and p.fixed_phase == 1
    assert p.rows_per_tile == 32 * 1024 // 1600 == 20 and p.tail_rows == 4725 % 20
    # a pitched [B, S, H, D] side (rows of 8 * 100 + 4 elements): the per-piece
    # form, units of 16 KB (10 rows)
    rc, p, _ = plan_ex(8, 2, 4725, 8, 100, 8 * 100 + 4, forced_path=PATH_STAGED)
    assert rc == OK and p.path == PATH_STAGED and p.vec_bytes == 8 and p.fixed_phase == 0
    assert p.rows_per_tile == 16 * 1024 // 1600 == 10 and p.tail_rows == 4725 % 10
    # one short-lived CTA per unit
    assert p.units == 8 * 2 * p.tiles_per_block and p.grid == p.units and p.block == 256
    cg = (10 * 200 + 30) // 16
    assert p.smem_bytes == (8 * 16 * (cg if cg % 2 else cg + 1) + 4 * 8 + 15) // 16 * 16
    # chunked: one plane per launch
    rc, p, _ = plan(8, 2, 4725, 8, 100, chunked=1, forced_path=PATH_STAGED)
    assert rc == OK and p.units == 8 * p.tiles_per_block and p.launches == 2
    # forced on an aligned shape, the pieces are 16 bytes
    rc, p, _ = plan(4, 1, 8192, 24, 128, forced_path=PATH_STAGED)
    assert rc == OK and p.path == PATH_STAGED and p.vec_bytes == 16
    # a row too long for the shared memory stays on the vector path
    rc, p, _ = plan(4, 1, 16, 4 * 8, 512, E=8)  # 8 groups x 32 KB runs (E = 8, D = 512)
    assert rc == OK and p.path == PATH_VEC
    rc, _, msg = plan(4, 1, 16, 4 * 8, 512, E=8, forced_path=PATH_STAGED)
    assert rc == ERR_UNSUPPORTED and "shared memory" in msg


def test_staged_fixed_phase_form():
    # a dense [B, S, H, D] side with gathered slabs at one offset: the fixed-
    # phase form (each thread's strided chunks share one phase within a row)
    for w, H, D, E, piece in ((4, 4, 3, 2, 2), (4, 4, 3, 4, 4), (2, 2, 5, 1, 1), (3, 3, 5, 2, 2),
                             (3, 6, 5, 2, 4)):
        for mode in (0, 1):
            rc, p, _ = plan(w, 2, 1000, H, D, mode=mode, E=E)
            assert rc == OK and p.path == PATH_STAGED and p.vec_bytes == piece
            assert p.fixed_phase == 1, (w, H, D, E, mode)
            rc, p, _ = plan(w, 2, 1000, H, D, mode=mode, E=E, forced_path=PATH_STAGED)
            assert rc == OK and p.fixed_phase == 1
    # units of 32 KB of strided rows (6-byte runs, 24-byte rows), one CTA
    # each; with at most 4 regions they sit 128 bytes apart
    rc, p, _ = plan(4, 1, 100000, 4, 3)
    assert p.rows_per_tile == 32 * 1024 // 24 and p.grid == p.units == 4 * p.tiles_per_block
    cg = (p.rows_per_tile * 6 + 30) // 16
    assert p.smem_bytes == (4 * 16 * ((cg + 7) // 8 * 8) + 4 * 4 + 15) // 16 * 16
    # with more regions, an odd number of 16-byte chunks apart
    rc, p, _ = plan(8, 1, 100000, 8, 3)
    cg = (p.rows_per_tile * 6 + 30) // 16
    assert p.fixed_phase == 1 and p.rows_per_tile == 32 * 1024 // 48
    assert p.smem_bytes == (8 * 16 * (cg if cg % 2 else cg + 1) + 4 * 8 + 15) // 16 * 16
    # gathered slabs at one offset past 16 bytes, strided slabs at others
    w, B, S, H, D, E = 4, 1, 64, 4, 3, 2
    ins, outs = fake_slabs(w, B * S * H * D * E)
    rc, p, _ = ulysses_a2a_plan([a + 2 * k for k, a in enumerate(ins)], [a + 6 for a in outs],
                                B, S, H, D, w, 0, 0, E)
    assert rc == OK and p.path == PATH_STAGED and p.fixed_phase == 1
    # the per-piece form when asked for
    rc, p, _ = plan(4, 2, 1000, 4, 3, staged_form=1)
    assert rc == OK and p.path == PATH_STAGED and p.fixed_phase == 0
    assert p.rows_per_tile == 16 * 1024 // 24
    # gathered slabs at different offsets: per-piece form
    rc, p, _ = ulysses_a2a_plan(ins, [a + 2 * k for k, a in enumerate(outs)], B, S, H, D, w, 0, 0, E)
    assert rc == OK and p.path == PATH_STAGED and p.vec_bytes == 2 and p.fixed_phase == 0
    rc, p, _ = ulysses_a2a_plan([a + 2 * k for k, a in enumerate(outs)], ins, B, S, H, D, w, 1, 0, E)
    assert rc == OK and p.path == PATH_STAGED and p.fixed_phase == 0
    # a pitched [B, S, H, D] side: per-piece form
    rc, p, _ = plan_ex(4, 2, 37, 4, 3, 4 * 3 + 1)
    assert rc == OK and p.path == PATH_STAGED and p.fixed_phase == 0
    # 16-byte pieces (forced on an aligned shape): per-piece form
    rc, p, _ = plan(4, 1, 8192, 24, 128, forced_path=PATH_STAGED)
    assert rc == OK and p.vec_bytes == 16 and p.fixed_phase == 0
    # rows whose phase period exceeds 256 chunks leave no thread a fixed phase:
    # 261-byte rows take the per-piece form; 87-byte rows (period 87, 2 * 87 =
    # 174 threads move chunks) and 81-byte rows (3 * 81 = 243) the fixed-phase one
    rc, p, _ = plan(3, 1, 64, 3, 87, E=1)
    assert rc == OK and p.path == PATH_STAGED and p.fixed_phase == 0
    for D in (29, 27):
        rc, p, _ = plan(3, 1, 64, 3, D, E=1)
        assert rc == OK and p.path == PATH_STAGED and p.fixed_phase == 1
    # the VEC and TMA paths never set it (8-byte vectors on a pitched side)
    rc, p, _ = plan(4, 1, 8192, 24, 128)
    assert rc == OK and p.path == PATH_TMA and p.fixed_phase == 0
    rc, p, _ = plan_ex(8, 2, 4725, 8, 100, 8 * 100 + 4)
    assert rc == OK and p.path == PATH_VEC and p.vec_bytes == 8 and p.fixed_phase == 0


def test_vec_when_misaligned_pointer():
    w, B, S, H, D, E = 2, 1, 8, 4, 64, 2
    ins, outs = fake_slabs(w, B * S * H * D * E)
    outs[1] += 8
    rc, p, _ = ulysses_a2a_plan(ins, outs, B, S, H, D, w, 0, 0, E)
    assert rc == OK and p.path == PATH_VEC and p.vec_bytes == 8     # 8-byte vectors: VEC
    outs[1] += 2
    rc, p, _ = ulysses_a2a_plan(ins, outs, B, S, H, D, w, 0, 0, E)
    assert rc == OK and p.path == PATH_STAGED and p.vec_bytes == 2  # 2-byte pieces: staged
    assert p.peeled == 0                                            # (offsets differ)
    rc, p, _ = ulysses_a2a_plan(ins, outs, B, S, H, D, w, 0, 0, E, forced_path=PATH_VEC)
    assert rc == OK and p.path == PATH_VEC and p.vec_bytes == 2
    outs[1] -= 2
    rc, p, msg = ulysses_a2a_plan(ins, outs, B, S, H, D, w, 0, 0, E, forced_path=PATH_TMA)
    assert rc == ERR_UNSUPPORTED and "aligned" in msg


def test_runs_at_one_offset_are_peeled():
    # slabs that all start the same number of bytes past a 16-byte boundary,
    # runs and rows of whole 16-byte multiples: every run starts at that offset
    # on both sides, so the vector kernel moves its 16-byte vectors between a
    # peeled head and tail
    w, B, S, H, D, E = 4, 2, 45, 8, 64, 2             # 256-byte runs
    for off in (2, 4, 6, 8, 10, 14):
        for mode in (0, 1):
            ins, outs = fake_slabs(w, B * S * H * D * E)
            ins, outs = [a + off for a in ins], [a + off for a in outs]
            rc, p, _ = ulysses_a2a_plan(ins, outs, B, S, H, D, w, mode, 0, E)
            assert rc == OK and p.path == PATH_VEC and p.vec_bytes == 16 and p.peeled == 1
            assert p.grid == p.units                  # one CTA per unit
            rc, p, _ = ulysses_a2a_plan(ins, outs, B, S, H, D, w, mode, 1, E)
            assert rc == OK and p.peeled == 1 and p.launches == B and p.grid == p.units
            # forced staged stays staged; forced VEC takes the windows too
            rc, p, _ = ulysses_a2a_plan(ins, outs, B, S, H, D, w, mode, 0, E,
                                        forced_path=PATH_STAGED)
            assert rc == OK and p.path == PATH_STAGED and p.peeled == 0
            rc, p, _ = ulysses_a2a_plan(ins, outs, B, S, H, D, w, mode, 0, E, forced_path=PATH_VEC)
            assert rc == OK and p.path == PATH_VEC and p.peeled == 1
            # one slab off by another amount: offsets no longer match
            outs[w - 1] += 2
            rc, p, _ = ulysses_a2a_plan(ins, outs, B, S, H, D, w, mode, 0, E)
            assert rc == OK and p.peeled == 0 and p.vec_bytes == 2
    # aligned slabs keep whole 16-byte vectors (nothing to peel)
    rc, p, _ = plan(4, 2, 45, 8, 64, forced_path=PATH_VEC)
    assert rc == OK and p.vec_bytes == 16 and p.peeled == 0
    # runs shorter than 64 bytes are not peeled
    ins, outs = fake_slabs(2, 2 * 9 * 2 * 32 * 2)
    ins, outs = [a + 2 for a in ins], [a + 2 for a in outs]
    rc, p, _ = ulysses_a2a_plan(ins, outs, 2, 9, 2, 24, 2, 0, 0, 2)      # 48-byte runs
    assert rc == OK and p.peeled == 0 and p.path == PATH_STAGED
    rc, p, _ = ulysses_a2a_plan(ins, outs, 2, 9, 2, 32, 2, 0, 0, 2)      # 64-byte runs
    assert rc == OK and p.peeled == 1
    # runs whose offsets drift from row to row (66-byte runs in 132-byte rows,
    # E = 1; 300-byte runs at w = 1) are not peeled
    ins, outs = fake_slabs(2, 2 * 11 * 4 * 33)
    rc, p, _ = ulysses_a2a_plan([a + 5 for a in ins], [a + 5 for a in outs], 2, 11, 4, 33, 2, 0,
                                0, 1)
    assert rc == OK and p.peeled == 0
    ins, outs = fake_slabs(1, 2 * 9 * 4 * 40 * 2)
    rc, p, _ = ulysses_a2a_plan([ins[0] + 10], [outs[0] + 10], 2, 9, 3, 50, 1, 0, 0, 2)
    assert rc == OK and p.peeled == 0 and p.row_bytes == 300
    rc, p, _ = ulysses_a2a_plan([ins[0] + 10], [outs[0] + 10], 2, 9, 4, 40, 1, 0, 0, 2)
    assert rc == OK and p.peeled == 1 and p.row_bytes == 320


def test_inputs_and_outputs_at_two_offsets_are_shifted():
    # the input slabs share one offset past a 16-byte boundary, the outputs
    # another: peeled = 2 (each destination vector joined from two aligned
    # source vectors), for every pair of different offsets
    w, B, S, H, D, E = 4, 2, 45, 8, 64, 2
    ins, outs = fake_slabs(w, B * S * H * D * E, gap=256)
    for a_in in range(0, 16, 2):
        for a_out in range(0, 16, 2):
            if a_in == a_out:
                continue
            for mode in (0, 1):
                rc, p, _ = ulysses_a2a_plan([a + a_in for a in ins], [a + a_out for a in outs],
                                            B, S, H, D, w, mode, 0, E)
                assert rc == OK and p.path == PATH_VEC and p.vec_bytes == 16 and p.peeled == 2
                assert p.grid == p.units
    # one output off by a third amount: no shared output offset, so staged
    o2 = [a + 4 for a in outs]
    o2[1] += 2
    rc, p, _ = ulysses_a2a_plan([a + 2 for a in ins], o2, B, S, H, D, w, 0, 0, E)
    assert rc == OK and p.peeled == 0 and p.path == PATH_STAGED
    # forced staged stays staged; runs under 64 bytes are not shifted
    rc, p, _ = ulysses_a2a_plan([a + 2 for a in ins], outs, B, S, H, D, w, 0, 0, E,
                                forced_path=PATH_STAGED)
    assert rc == OK and p.path == PATH_STAGED
    ins2, outs2 = fake_slabs(2, 2 * 9 * 2 * 24 * 2, gap=256)
    rc, p, _ = ulysses_a2a_plan([a + 2 for a in ins2], outs2, 2, 9, 2, 24, 2, 0, 0, 2)
    assert rc == OK and p.peeled == 0


def test_peeled_pitched_and_packed_plans():
    # q of a packed [B, S, 3, H, D] buffer 6 bytes past a boundary, the dense
    # side 6 bytes past too (rows of 3*H*D*E bytes, a multiple of 16): peeled
    w, B, S, H, D, E = 4, 2, 37, 8, 64, 2
    pitch = 3 * H * D
    rc, p, _ = plan_ex(w, B, S, H, D, pitch, base=(1 << 40) + 6)
    assert rc == OK and p.path == PATH_VEC and p.peeled == 1 and p.row_pitch == pitch
    # a pitch that moves the offset by 4 bytes per row: not peeled
    rc, p, _ = plan_ex(w, B, S, H, D, pitch + 2, base=(1 << 40) + 6)
    assert rc == OK and p.peeled == 0
    # T = 3 head-packed tensors, every slab 2 bytes off
    step = (B * S * 3 * H * D * E + 4095) // 4096 * 4096
    strided = [(1 << 40) + 2 + k * step for k in range(w)]
    gathered = [(1 << 44) + 2 + k * step for k in range(3 * w)]
    for mode in (0, 1):
        ins, outs = (strided, gathered) if mode == 0 else (gathered, strided)
        rc, p, _ = _lib.ulysses_a2a_plan_ex(ins, outs, B, S, H, D, w, mode, 0, E, ntensors=3)
        assert rc == OK and p.path == PATH_VEC and p.peeled == 1


def test_vec_when_too_many_ranks_for_tma():
    rc, p, _ = plan(16, 1, 32, 16, 64)
    assert rc == OK and p.path == PATH_VEC and p.vec_bytes == 16
    rc, p, msg = plan(16, 1, 32, 16, 64, forced_path=PATH_TMA)
    assert rc == ERR_UNSUPPORTED


def test_vec_when_box_dim_too_large():
    rc, p, _ = plan(2, 1, 8, 2, 512)            # D = 512 > 256
    assert rc == OK and p.path == PATH_VEC


def test_forced_vec_geometry():
    rc, p, _ = plan(4, 1, 8192, 24, 128, forced_path=PATH_VEC)
    assert rc == OK and p.path == PATH_VEC and p.vec_bytes == 16
    # 12 KB units of 8 rows x 1536 B: 16 blocks x 1024 tiles, one CTA per unit
    assert p.rows_per_tile == 12 * 1024 // 1536 == 8 and p.units == 16 * 1024
    assert p.block == 256 and p.grid == p.units
    assert p.producers == 0 and p.lookahead == 0


def test_vec_grid_one_cta_per_unit_unless_set():
    rc, p, _ = plan(8, 2, 4725, 40, 128, forced_path=PATH_VEC)      # 1280 B rows
    assert rc == OK and p.rows_per_tile == 9 and p.tail_rows == 4725 % 9
    assert p.units == 8 * 2 * 8 * 525 and p.grid == p.units
    # a row longer than the target makes one-row units
    rc, p, _ = plan(1, 1, 100, 64, 128, forced_path=PATH_VEC)       # 16 KB rows
    assert rc == OK and p.rows_per_tile == 1 and p.units == 100 and p.grid == 100
    # ctas_per_sm selects a grid-stride grid; rows_per_tile is kept as given
    rc, p, _ = plan(2, 1, 8192, 24, 128, forced_path=PATH_VEC, rows_per_tile=21, ctas_per_sm=16)
    assert rc == OK and p.rows_per_tile == 21 and p.units == 4 * 391 and p.grid == 1564
    rc, p, _ = plan(8, 2, 4725, 40, 128, forced_path=PATH_VEC, ctas_per_sm=4)
    assert rc == OK and p.grid == 148 * 4


def test_tuning_knobs():
    rc, p, _ = plan(4, 1, 8192, 24, 128, rows_per_tile=16, stages=4, ctas_per_sm=2,
                    chunk_units=0)
    assert rc == OK and p.rows_per_tile == 16 and p.stages == 4 and p.grid == 296
    assert p.smem_bytes == 4 * 24 * 1024
    rc, p, _ = plan(4, 1, 8192, 24, 128, producers=2, chunk_units=7, order=0)
    assert rc == OK and (p.producers, p.chunk_units, p.order) == (2, 7, 0)
    assert p.grid == -(-p.units // 7)


@pytest.mark.parametrize("knob,value", [("rows_per_tile", 257), ("rows_per_tile", -1),
                                        ("ctas_per_sm", 33), ("stages", 33), ("producers", 9),
                                        ("order", 2), ("chunk_units", -2), ("lookahead", -1),
                                        ("host_chunks", 65), ("host_chunks", -1),
                                        ("staged_form", 2), ("staged_form", -1)])
def test_tuning_out_of_range_is_rejected(knob, value):
    rc, _, msg = plan(4, 1, 64, 8, 64, **{knob: value})
    assert rc == ERR_INVALID and knob in msg


def test_tuning_struct_layout():
    assert ctypes.sizeof(_lib.TuningT) == 36


def test_ring_split_between_producers_loads_and_stores():
    # stages split evenly over up to 4 producer warps (sub-rings of >= 2);
    # per producer L loads in flight, sp - L stores allowed to read their stages
    for S, np_, sp, L in [(2, 1, 2, 1), (3, 1, 3, 2), (4, 2, 2, 1), (6, 3, 2, 1), (8, 4, 2, 1),
                          (12, 4, 3, 2), (16, 4, 4, 2), (32, 4, 8, 4)]:
        rc, p, _ = plan(4, 1, 8192, 24, 128, rows_per_tile=4, stages=S, chunk_units=0)
        assert rc == OK, S
        assert (p.producers, p.stages // p.producers, p.lookahead) == (np_, sp, L), S
        assert p.stages == np_ * sp and p.block == 32 * np_
        assert 1 <= p.lookahead < p.stages // p.producers


def test_large_rows_reduce_stages_then_producers():
    # 24 KB rows: four producers keep two 24 KB stages each (192 KB)
    # persistent schedule
    rc, p, _ = plan(2, 1, 16, 128, 192, chunk_units=0, forced_path=PATH_TMA)
    assert rc == OK and p.path == PATH_TMA and p.rows_per_tile == 1
    assert p.row_bytes == 24 * 1024
    assert (p.producers, p.stages, p.smem_bytes) == (4, 8, 192 * 1024)
    # 32 KB rows: two stages for four producers would not fit; three producers do
    rc, p, _ = plan(2, 1, 16, 128, 256, chunk_units=0, forced_path=PATH_TMA)
    assert rc == OK and p.row_bytes == 32 * 1024
    assert (p.producers, p.stages, p.smem_bytes) == (3, 6, 192 * 1024)
    # 64 KB rows: one producer with a three-stage ring
    rc, p, _ = plan(2, 1, 8, 256, 256, chunk_units=0, forced_path=PATH_TMA)
    assert rc == OK and p.path == PATH_TMA and p.row_bytes == 64 * 1024
    assert (p.producers, p.stages, p.lookahead, p.smem_bytes) == (1, 3, 2, 192 * 1024)
    # default (chunked grid): one producer, one tile; the residency cap reserves
    # shared memory for round(100 KB / tile) CTAs per SM (24 KB tiles: 4 CTAs)
    rc, p, _ = plan(2, 1, 16, 128, 192, forced_path=PATH_TMA)
    assert (p.producers, p.stages, p.chunk_units) == (1, 1, 1)
    assert p.smem_bytes == (228 * 1024 // 4 - 1024) // 1024 * 1024
    # 64 KB tiles: cap round(100 / 64) = 2 CTAs per SM (113 KB each)
    rc, p, _ = plan(2, 1, 8, 256, 256, forced_path=PATH_TMA)
    assert (p.producers, p.stages, p.chunk_units, p.smem_bytes) == (1, 1, 1, 113 * 1024)
    # a tile larger than the cap's share keeps its own size (cap 1 is 220 KB max)
    rc, p, _ = plan(2, 1, 8, 256, 256, ctas_per_sm=8, forced_path=PATH_TMA)
    assert p.smem_bytes == 64 * 1024


# ---- argument validation ----------------------------------------------------

@pytest.mark.parametrize("args,code", [
    (dict(w=2, B=1, S=4, H=3, D=8), ERR_INVALID),        # H % w
    (dict(w=2, B=-1, S=4, H=4, D=8), ERR_INVALID),
    (dict(w=2, B=1, S=-3, H=4, D=8), ERR_INVALID),
    (dict(w=2, B=1, S=4, H=4, D=-1), ERR_INVALID),
    (dict(w=0, B=1, S=4, H=4, D=8), ERR_INVALID),
    (dict(w=65, B=1, S=4, H=65, D=8), ERR_INVALID),
    (dict(w=2, B=1, S=4, H=4, D=8, mode=2), ERR_INVALID),
    (dict(w=2, B=1, S=4, H=4, D=8, chunked=3), ERR_INVALID),
    (dict(w=2, B=1, S=4, H=4, D=8, chunked=-1), ERR_INVALID),
    (dict(w=2, B=1, S=4, H=4, D=8, E=3), ERR_INVALID),
])
def test_rejects_bad_arguments(args, code):
    a = dict(args)
    w = a.pop("w")
    B, S, H, D = a.pop("B"), a.pop("S"), a.pop("H"), a.pop("D")
    mode, chunked, E = a.pop("mode", 0), a.pop("chunked", 0), a.pop("E", 2)
    ins, outs = fake_slabs(max(w, 1), max(B * S * H * D * E, 1))
    rc, _, msg = ulysses_a2a_plan(ins[:max(w, 0)] or [0], outs[:max(w, 0)] or [0], B, S, H, D, w,
                                  mode, chunked, E)
    assert rc == code and msg


@pytest.mark.parametrize("B,S,H,D", [(0, 4, 4, 8), (1, 0, 4, 8), (1, 4, 0, 8), (1, 4, 4, 0)])
def test_empty_relayout_is_a_no_op_plan(B, S, H, D):
    # any zero size: nothing to move, nothing to launch, NULL slabs accepted
    for chunked in (0, 1, 2):
        rc, p, msg = ulysses_a2a_plan([0, 0], [0, 0], B, S, H, D, 2, 0, chunked, 2)
        assert rc == OK, msg
        assert p.units == 0 and p.launches == 0 and p.payload_bytes == 0
    rc, _, _ = ulysses_a2a_plan([0, 0], [0, 0], B, S, 3, D, 2, 0, 0, 2)   # H % w still checked
    assert rc == ERR_INVALID


def test_rejects_size_overflow():
    ins, outs = fake_slabs(2, 16)
    rc, _, msg = ulysses_a2a_plan(ins, outs, 1 << 40, 1 << 20, 2, 8, 2, 0, 0, 2)
    assert rc == ERR_INVALID and "overflow" in msg


def test_rejects_null_pointers():
    rc, _, _ = ulysses_a2a_plan(None, None, 1, 1, 2, 1, 2, 0, 0, 2)
    assert rc == ERR_INVALID
    ins, outs = fake_slabs(2, 64)
    ins[1] = 0
    rc, _, msg = ulysses_a2a_plan(ins, outs, 1, 4, 2, 4, 2, 0, 0, 2)
    assert rc == ERR_INVALID and "NULL" in msg


def test_rejects_output_overlapping_input():
    w, B, S, H, D, E = 2, 1, 4, 4, 8, 2
    nbytes = B * S * H * D * E
    ins, outs = fake_slabs(w, nbytes)
    outs[0] = ins[1] + nbytes - 2             # last element of input 1 shared
    rc, _, msg = ulysses_a2a_plan(ins, outs, B, S, H, D, w, 0, 0, E)
    assert rc == ERR_OVERLAP and "input" in msg
    outs[0] = ins[1] + nbytes                 # touching but disjoint: fine
    outs[1] = outs[0] + nbytes
    rc, _, _ = ulysses_a2a_plan(ins, outs, B, S, H, D, w, 0, 0, E)
    assert rc == OK


def test_rejects_outputs_overlapping_each_other_and_in_place():
    w, B, S, H, D, E = 2, 1, 4, 4, 8, 2
    nbytes = B * S * H * D * E
    ins, outs = fake_slabs(w, nbytes)
    outs[1] = outs[0] + 16
    rc, _, msg = ulysses_a2a_plan(ins, outs, B, S, H, D, w, 0, 0, E)
    assert rc == ERR_OVERLAP and "output" in msg
    rc, _, _ = ulysses_a2a_plan(ins, ins, B, S, H, D, w, 0, 0, E)   # in place
    assert rc == ERR_OVERLAP


def test_inputs_may_alias_each_other():
    w, B, S, H, D, E = 2, 1, 4, 4, 8, 2
    ins, outs = fake_slabs(w, B * S * H * D * E)
    ins[1] = ins[0]
    rc, _, _ = ulysses_a2a_plan(ins, outs, B, S, H, D, w, 0, 0, E)
    assert rc == OK


# ---- entry points that need no GPU ------------------------------------------

def test_null_context_handling():
    lib = _lib.lib
    assert lib.ulysses_a2a_destroy(None) == OK
    assert lib.ulysses_a2a_launch_count(None) == 0
    assert lib.ulysses_a2a_last_error(None) == b"NULL context"
    assert lib.ulysses_a2a_set_path(None, PATH_AUTO) == ERR_INVALID
    assert lib.ulysses_a2a_set_tuning(None, None) == ERR_INVALID
    arr = _lib.ptr_array([1, 2])
    assert lib.ulysses_a2a_run(None, arr, arr, 1, 1, 2, 1, 2, 0, 0, None) == ERR_INVALID
    assert lib.ulysses_a2a_run_host(None, arr, arr, 1, 1, 2, 1, 2, 0, 0, None) == ERR_INVALID
    assert lib.ulysses_a2a_status(None, None) == ERR_INVALID


def test_create_rejects_bad_element_size_before_touching_cuda():
    h = ctypes.c_void_p()
    assert _lib.lib.ulysses_a2a_create(ctypes.byref(h), 0, 3) == ERR_INVALID
    assert _lib.lib.ulysses_a2a_create(None, 0, 2) == ERR_INVALID


# ---- row pitch on the [B, S, H, D] side (packed QKV layouts) -----------------

def plan_ex(w, B, S, H, D, pitch, mode=0, E=2, base=1 << 40, **kw):
    ext = ((B * S - 1) * pitch + H * D) * E
    dense = B * S * H * D * E
    step = (max(ext, dense) + 4095) // 4096 * 4096
    ins = [base + k * step for k in range(w)]
    outs = [base + (w + k) * step for k in range(w)]
    return _lib.ulysses_a2a_plan_ex(ins, outs, B, S, H, D, w, mode, 0, E, row_pitch=pitch, **kw)


def test_pitch_defaults_to_dense_and_is_reported():
    rc, p, _ = plan_ex(4, 1, 64, 8, 64, 0)
    assert rc == OK and p.row_pitch == 8 * 64
    rc, p, _ = plan_ex(4, 1, 64, 8, 64, 3 * 8 * 64, forced_path=PATH_TMA)
    assert rc == OK and p.row_pitch == 3 * 8 * 64 and p.path == PATH_TMA


def test_pitch_smaller_than_a_row_is_rejected():
    rc, _, msg = plan_ex(4, 1, 64, 8, 64, 8 * 64 - 1)
    assert rc == ERR_INVALID and "pitch" in msg


def test_pitch_alignment_selects_the_vector_width():
    # pitch * E = (512 + 4) * 2 bytes: 8-byte aligned rows only
    rc, p, _ = plan_ex(4, 1, 64, 8, 64, 8 * 64 + 4)
    assert rc == OK and p.path == PATH_VEC and p.vec_bytes == 8
    rc, p, _ = plan_ex(4, 1, 64, 8, 64, 8 * 64 + 2)          # 4-byte aligned rows: staged
    assert rc == OK and p.path == PATH_STAGED and p.vec_bytes == 4
    rc, p, _ = plan_ex(4, 1, 64, 8, 64, 8 * 64 + 2, forced_path=PATH_VEC)
    assert rc == OK and p.path == PATH_VEC and p.vec_bytes == 4
    rc, _, msg = plan_ex(4, 1, 64, 8, 64, 8 * 64 + 4, forced_path=PATH_TMA)
    assert rc == ERR_UNSUPPORTED and "pitch" in msg


def test_pitched_extent_counts_for_overlap():
    # mode 1 writes pitched outputs: a second output placed inside the first
    # one's gaps still overlaps its extent
    w, B, S, H, D, E = 2, 1, 4, 4, 8, 2
    pitch = 3 * H * D
    ins = [1 << 40, (1 << 40) + (1 << 20)]
    outs = [(1 << 41), (1 << 41) + H * D * E]          # interleaved like k next to q
    rc, _, msg = _lib.ulysses_a2a_plan_ex(ins, outs, B, S, H, D, w, 1, 0, E, row_pitch=pitch)
    assert rc == ERR_OVERLAP
    # the same pointers as *inputs* of mode 0 may alias (q, k, v of one buffer)
    rc, _, _ = _lib.ulysses_a2a_plan_ex(outs, [1 << 42, (1 << 42) + (1 << 20)], B, S, H, D, w, 0,
                                        0, E, row_pitch=pitch)
    assert rc == OK


# ---- test-only environment overrides at context creation ----------------------

@pytest.mark.parametrize("name,value", [("ULYSSES_A2A_FORCE_PATH", "fast"),
                                        ("ULYSSES_A2A_CTAS_PER_SM", "0"),
                                        ("ULYSSES_A2A_CTAS_PER_SM", "33"),
                                        ("ULYSSES_A2A_CTAS_PER_SM", "8x")])
def test_malformed_environment_override_fails_creation(monkeypatch, name, value):
    monkeypatch.setenv(name, value)
    h = ctypes.c_void_p()
    # checked before the device is touched, so this holds without a GPU too
    assert _lib.lib.ulysses_a2a_create(ctypes.byref(h), 0, 2) == ERR_INVALID
    assert not h.value


def test_valid_environment_override_is_accepted(monkeypatch):
    monkeypatch.setenv("ULYSSES_A2A_FORCE_PATH", "vec")
    monkeypatch.setenv("ULYSSES_A2A_CTAS_PER_SM", "8")
    h = ctypes.c_void_p()
    rc = _lib.lib.ulysses_a2a_create(ctypes.byref(h), 0, 2)
    assert rc != ERR_INVALID               # OK on a GPU, ERR_DEVICE without one
    if rc == OK:
        assert _lib.ulysses_a2a_get_settings(h)[:2] == (OK, PATH_VEC)
        _lib.ulysses_a2a_destroy(h)


def test_get_settings_rejects_null_context():
    assert _lib.lib.ulysses_a2a_get_settings(None, None, None) == ERR_INVALID


# ---- head-packed tensors in one launch (ntensors) -----------------------------

def packed_plan(T, w, B, S, H, D, mode=0, chunked=0, E=2, **kw):
    P = B * S * H * D * E
    strided = [(1 << 40) + k * (1 << 32) for k in range(w)]
    # the gathered side has max(T, 1) * w slabs (ntensors 0 means one tensor)
    gathered = [(1 << 44) + k * (1 << 32) for k in range(max(T, 1) * w)]
    ins, outs = (strided, gathered) if mode == 0 else (gathered, strided)
    return _lib.ulysses_a2a_plan_ex(ins, outs, B, S, H, D, w, mode, chunked, E, ntensors=T, **kw)


def test_packed_plan_geometry():
    rc, p, msg = packed_plan(3, 4, 2, 8192, 24, 128)
    assert rc == OK, msg
    assert p.path == PATH_VEC and p.row_bytes == 6 * 128 * 2
    assert p.row_pitch == 3 * 24 * 128                    # one packed row holds q, k and v
    assert p.units == 3 * 4 * 4 * 2 * p.tiles_per_block    # T*w head groups x w blocks x planes
    assert p.payload_bytes == 3 * 4 * 2 * 8192 * 24 * 128 * 2
    # ntensors 0 and 1 both mean one tensor, and plan exactly as before
    rc0, p0, _ = packed_plan(0, 4, 2, 8192, 24, 128)
    rc1, p1, _ = packed_plan(1, 4, 2, 8192, 24, 128)
    rcp, pp, _ = plan(4, 2, 8192, 24, 128)
    assert rc0 == rc1 == rcp == OK and p0.as_dict() == p1.as_dict() == pp.as_dict()


def test_packed_plan_validation():
    assert packed_plan(17, 4, 1, 64, 8, 64)[0] == ERR_INVALID        # T*w > 64
    assert packed_plan(-1, 4, 1, 64, 8, 64)[0] == ERR_INVALID
    assert packed_plan(3, 4, 1, 64, 8, 64, chunked=2)[0] == ERR_UNSUPPORTED
    rc, _, msg = packed_plan(3, 4, 1, 64, 8, 64, forced_path=PATH_TMA)
    assert rc == ERR_UNSUPPORTED and "packed" in msg
    # two gathered slabs of different tensors overlapping
    w, T, B, S, H, D = 2, 3, 1, 64, 4, 64
    slab = B * S * H * D * 2
    strided = [(1 << 40) + k * (1 << 32) for k in range(w)]
    gathered = [(1 << 44) + k * (1 << 32) for k in range(T * w)]
    gathered[5] = gathered[1] + slab // 2
    rc, _, msg = _lib.ulysses_a2a_plan_ex(strided, gathered, B, S, H, D, w, 0, 0, 2, ntensors=T)
    assert rc == ERR_OVERLAP
    # a NULL among the T*w mode-1 inputs
    gathered = [(1 << 44) + k * (1 << 32) for k in range(T * w)]
    gathered[4] = 0
    rc, _, msg = _lib.ulysses_a2a_plan_ex(gathered, strided, B, S, H, D, w, 1, 0, 2, ntensors=T)
    assert rc == ERR_INVALID and "NULL" in msg


@pytest.mark.parametrize("compiler,std", [("gcc", "c99"), ("gcc", "c11"), ("g++", "c++11"),
                                          ("g++", "c++17")])
def test_header_compiles_standalone(tmp_path, compiler, std):
    """The public header is self-contained C (and C++): it compiles on its own,
    pedantically, with every warning an error, and sizeof the ABI structs
    agrees with the Python mirrors."""
    import shutil
    import subprocess

    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not available")
    ext = "c" if compiler == "gcc" else "cpp"
    src = tmp_path / f"hdr.{ext}"
    src.write_text(
        '#include "ulysses_a2a.h"\n'
        "#include <stdio.h>\n"
        "int main(void) {\n"
        '  printf("%d %d %d %d\\n", (int)sizeof(ulysses_a2a_plan_t),\n'
        "         (int)sizeof(ulysses_a2a_tuning_t), (int)sizeof(ulysses_a2a_desc_t),\n"
        "         ULYSSES_A2A_PEER_HANDLE_BYTES);\n"
        "  return 0;\n"
        "}\n")
    exe = tmp_path / "hdr"
    subprocess.run([compiler, f"-std={std}", "-pedantic", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    assert [int(v) for v in out] == [ctypes.sizeof(_lib.PlanT), ctypes.sizeof(_lib.TuningT),
                                     ctypes.sizeof(_lib.DescT), _lib.PEER_HANDLE_BYTES]


# ---- planner invariants over random shapes (property test) -------------------

from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402


def _one_row_fits_stage(R, ng):
    """Whether one strided row fits the staged path's 96 KB of shared memory:
    ng regions of (R + 30) // 16 chunks, rounded to an odd count, plus ng
    4-byte region offsets."""
    cg = (R + 30) // 16
    return ng * 16 * (cg if cg % 2 else cg + 1) + 4 * ng <= 96 * 1024


@settings(max_examples=300, deadline=None, derandomize=True, database=None)
@given(w=st.sampled_from([1, 2, 3, 4, 8, 16]), hw=st.integers(1, 6), B=st.integers(1, 4),
       S=st.integers(1, 5000), D=st.sampled_from([1, 3, 8, 13, 64, 128, 256]),
       E=st.sampled_from([1, 2, 4, 8]), mode=st.sampled_from([0, 1]),
       chunked=st.sampled_from([0, 1]),
       path=st.sampled_from([PATH_AUTO, PATH_VEC, PATH_STAGED]),
       rows=st.sampled_from([0, 0, 1, 7, 64]), ntensors=st.sampled_from([1, 1, 2, 3]))
def test_planner_invariants(w, hw, B, S, D, E, mode, chunked, path, rows, ntensors):
    H = hw * w
    if ntensors * w > 64:
        return
    slab = B * S * H * D * E
    step = (slab * ntensors + 4095) // 4096 * 4096
    strided = [(1 << 40) + k * step for k in range(w)]
    gathered = [(1 << 44) + k * step for k in range(ntensors * w)]
    ins, outs = (strided, gathered) if mode == 0 else (gathered, strided)
    rc, p, msg = _lib.ulysses_a2a_plan_ex(ins, outs, B, S, H, D, w, mode, chunked, E,
                                          forced_path=path, ntensors=ntensors,
                                          rows_per_tile=rows)
    if path == PATH_STAGED and rc == ERR_UNSUPPORTED:
        assert "shared memory" in msg       # one strided row does not fit
        assert not _one_row_fits_stage(hw * D * E, ntensors * w)
        return
    assert rc == OK, msg
    nb = 1 if chunked else B
    if p.path == PATH_STAGED:
        # one unit per (b, j, tile), every head group of its rows; pieces of the
        # widest width the run and the pitch allow; shared memory within 96 KB
        assert path in (PATH_AUTO, PATH_STAGED)
        hde = ntensors * hw * w * D * E
        assert 1 <= p.rows_per_tile <= S and p.tiles_per_block == -(-S // p.rows_per_tile)
        assert p.rows_per_tile == 1 or p.rows_per_tile * hde <= (32 if p.fixed_phase else 16) * 1024 or rows
        assert p.units == w * nb * p.tiles_per_block and p.grid == p.units
        assert p.block == 256 and p.smem_bytes <= 96 * 1024
        v = p.vec_bytes
        assert p.row_bytes % v == 0 and (p.row_pitch * E) % v == 0
        assert v == 16 or (p.row_bytes % (2 * v) or (p.row_pitch * E) % (2 * v))
        if path == PATH_AUTO:
            assert v <= 4 or (v == 8 and p.fixed_phase)
        return
    # tiles cover every sequence row exactly once per (r, b, j) block
    assert 1 <= p.rows_per_tile <= min(S, 256)
    assert p.tiles_per_block == -(-S // p.rows_per_tile)
    assert p.tail_rows == S % p.rows_per_tile
    assert p.units == ntensors * w * w * nb * p.tiles_per_block
    assert p.payload_bytes == ntensors * w * slab
    assert p.launches == (B if chunked else 1)
    assert p.row_bytes == hw * D * E and p.row_pitch == ntensors * H * D
    if rows:
        # as requested, but never past the sequence, nor (TMA) past a 64 KB tile
        cap = max(1, 64 * 1024 // p.row_bytes) if p.path == PATH_TMA else rows
        assert p.rows_per_tile == min(rows, S, cap)
    if p.path == PATH_TMA:
        assert path == PATH_AUTO and ntensors == 1
        assert (D * E) % 16 == 0 and w <= 8 and D <= 256 and hw <= 256
        assert p.rows_per_tile * p.row_bytes <= 64 * 1024
        assert 32 <= p.block == 32 * p.producers <= 256
        assert p.smem_bytes <= 220 * 1024
        assert p.grid == -(-p.units // p.chunk_units)
    else:
        assert p.path == PATH_VEC and p.block == 256
        # 4 KiB-aligned slabs share no offset past a 16-byte boundary: never peeled
        assert p.peeled == 0
        assert p.grid == p.units
        v = p.vec_bytes
        assert v in (1, 2, 4, 8, 16) and p.row_bytes % v == 0 and (p.row_pitch * E) % v == 0
        # AUTO leaves narrower vectors to the staged path unless a row is too long,
        # and 8-byte vectors to its fixed-phase form where that applies
        assert path == PATH_VEC or v >= 8 or not _one_row_fits_stage(hw * D * E, ntensors * w)
        if path == PATH_AUTO and v == 8:
            rc2, p2, _ = _lib.ulysses_a2a_plan_ex(ins, outs, B, S, H, D, w, mode, chunked, E,
                                                  forced_path=PATH_STAGED, ntensors=ntensors,
                                                  rows_per_tile=rows)
            assert rc2 != OK or p2.fixed_phase == 0
        # the widest width the run length and the pitch allow (pointers are 4 KiB aligned)
        assert v == 16 or (p.row_bytes % (2 * v) or (p.row_pitch * E) % (2 * v))
