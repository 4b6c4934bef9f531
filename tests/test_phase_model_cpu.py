"""A CPU model of the staged path's fixed-phase kernel (kernels_phase.cuh): its
index arithmetic replayed at the byte level, no GPU needed.

The kernel moves a unit's strided segment (rows of HDE = ng*R bytes, dense) as
16-byte chunks c = t + m*nthr per thread t, with nthr a multiple of
HDE / gcd(HDE, 16); each thread works out the shared-memory offsets of its
chunk's pieces once per unit. This model restates those formulas (the row and
phase of a thread's first chunk, the piece offsets, the per-chunk step) and
checks, for units of many shapes and offsets:
- every region byte [a_g, a_g + rows*R) of every region is written exactly
  once, from the segment byte the element map names (region g holds head
  group g: row i, byte col at a_g + i*R + col);
- every shared access stays inside its region;
- mode 1's load batches: the strided chunks assembled before the second wait
  (c < cA) read only region chunks of the first batch (whole 8-chunk blocks up
  to cgA8), and each thread issues all its first-batch chunks before any of
  the second.
The model is checked against the element map, not against the GPU; the GPU
tests compare the kernel itself with the oracle.
"""

import math
import random

import pytest


def phase_movers(HDE, block=256):
    g = 16
    while HDE % g:
        g >>= 1
    period = HDE // g
    return period * (block // period) if period <= block else 0


def region_stride(R, ng, S_tile):
    Cg = (S_tile * R + 30) // 16
    chunks = (Cg + 7) // 8 * 8 if ng <= 4 else (Cg if Cg % 2 else Cg + 1)
    return Cg, 16 * chunks


def piece_offsets(G, kap, R, RS, ng):
    g, col, dr, off = kap // R, kap % R, 0, []
    for _ in range(16 // G):
        off.append(g * RS + dr * R + col)
        col += G
        if col == R:
            col, g = 0, g + 1
            if g == ng:
                g, dr = 0, dr + 1
    return off


def replay_unit(R, ng, G, rows, S_tile, a_s, a_g):
    HDE = ng * R
    Cg, RS = region_stride(R, ng, S_tile)
    nthr = phase_movers(HDE)
    assert nthr >= 128 and (16 * nthr) % HDE == 0
    step_rows = 16 * nthr // HDE
    segB, L = rows * HDE, rows * R
    nS = (a_s + segB + 15) >> 4
    rowsA = rows >> 1
    cgA = (a_g + rowsA * R + 15) >> 4
    cgA8 = (cgA + 7) & ~7
    cA = (a_s + rowsA * HDE) >> 4
    written = {}
    for tid in range(nthr):
        o_first = 16 * tid - a_s
        i0 = (o_first + 16 * HDE) // HDE - 16           # floor(o_first / HDE)
        assert i0 == math.floor(o_first / HDE)
        kap = o_first - i0 * HDE
        base0 = a_g + i0 * R
        off = piece_offsets(G, kap, R, RS, ng)
        m = 0
        while tid + m * nthr < nS:
            c = tid + m * nthr
            o = 16 * c - a_s
            x0, x1 = (-o if o < 0 else 0), min(16, segB - o)
            for n in range(16 // G):
                if not (x0 <= n * G < x1):
                    continue
                pos = base0 + m * step_rows * R + off[n]
                g, r = divmod(pos, RS)
                assert a_g <= r and r + G <= a_g + L, "a piece outside its region's range"
                if c < cA:
                    assert r // 16 < cgA8, "gathered before its load batch landed"
                for b in range(G):
                    assert pos + b not in written, "a region byte written twice"
                    written[pos + b] = o + n * G + b
            m += 1
    assert len(written) == segB
    for g in range(ng):
        for i in range(rows):
            for col in range(R):
                assert written[g * RS + a_g + i * R + col] == (i * ng + g) * R + col
    # the region chunks a thread issues for mode 1, in its order: whole blocks
    # of the first batch before any of the second
    for tid in range(256):
        second = False
        for e in range(tid, ng * ((Cg + 7) & ~7), 256):
            q = e >> 3
            c = (q // ng) * 8 + (e & 7)
            if c >= cgA8:
                second = True
            else:
                assert not second


SHAPES = [(6, 2), (12, 4), (3, 1), (10, 2), (5, 1), (20, 4), (24, 8), (36, 4), (8, 8),
          (1, 1), (7, 1), (200, 8), (2, 2)]


@pytest.mark.parametrize("R,G", SHAPES, ids=lambda v: str(v))
def test_fixed_phase_piece_placement(R, G):
    rng = random.Random(1000 + R)
    cases = 0
    for ng in (1, 2, 3, 4, 6, 8, 16, 24, 27, 35, 64):
        if phase_movers(ng * R) < 128:
            continue
        for _ in range(3):
            S_tile = rng.choice([1, 2, 3, 5, 64, max(1, 32768 // (ng * R))])
            rows = rng.randint(1, S_tile)
            replay_unit(R, ng, G, rows, S_tile, rng.randrange(0, 16, G), rng.randrange(0, 16, G))
            cases += 1
    assert cases > 0


def test_mover_count_is_a_multiple_of_the_phase_period():
    for HDE in range(1, 4097):
        n = phase_movers(HDE)
        period = HDE // math.gcd(HDE, 16)
        assert n % period == 0 if n else period > 256
        assert n == 0 or 256 - period < n <= 256


def test_model_geometry_matches_the_planner():
    # the model's unit rows and region stride are the ones the library plans
    from sequence_all_re_b200 import _lib
    for w, H, D, E in ((4, 4, 3, 2), (8, 8, 3, 2), (16, 16, 3, 2), (3, 3, 5, 2), (4, 4, 3, 4),
                       (2, 2, 5, 1), (4, 8, 5, 2), (8, 8, 9, 4)):
        B, S = 1, 100000
        R, ng = (H // w) * D * E, w
        slab = B * S * H * D * E
        step = (slab + 4095) // 4096 * 4096
        ins = [(1 << 40) + k * step for k in range(w)]
        outs = [(1 << 44) + k * step for k in range(w)]
        rc, p, msg = _lib.ulysses_a2a_plan(ins, outs, B, S, H, D, w, 0, 0, E)
        assert rc == _lib.OK and p.path == _lib.PATH_STAGED and p.fixed_phase == 1, msg
        assert p.rows_per_tile == 32768 // (ng * R)
        _, RS = region_stride(R, ng, p.rows_per_tile)
        assert p.smem_bytes == (ng * RS + 4 * ng + 15) // 16 * 16
