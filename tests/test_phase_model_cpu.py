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
  the second;
- mode 0 with pieces of 4 bytes or more (gather form): the segment's chunks
  occupy distinct places of the swizzled image, every gathered byte comes from
  the segment byte the element map names, exactly once, and the chunks built
  before the second wait read only image chunks of the first load batch.
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
    # the model's unit rows, region stride and mode-0 image are the ones the
    # library plans (mode 0 with pieces of 4 bytes or more: the image only)
    from sequence_all_re_b200 import _lib
    for w, H, D, E in ((4, 4, 3, 2), (8, 8, 3, 2), (16, 16, 3, 2), (3, 3, 5, 2), (4, 4, 3, 4),
                       (2, 2, 5, 1), (4, 8, 5, 2), (8, 8, 9, 4), (4, 4, 4, 2)):
        B, S = 1, 100000
        R, ng = (H // w) * D * E, w
        slab = B * S * H * D * E
        step = (slab + 4095) // 4096 * 4096
        strided = [(1 << 40) + k * step for k in range(w)]
        gathered = [(1 << 44) + k * step for k in range(w)]
        for mode in (0, 1):
            ins, outs = (strided, gathered) if mode == 0 else (gathered, strided)
            rc, p, msg = _lib.ulysses_a2a_plan(ins, outs, B, S, H, D, w, mode, 0, E)
            assert rc == _lib.OK and p.path == _lib.PATH_STAGED and p.fixed_phase == 1, msg
            assert p.rows_per_tile == 32768 // (ng * R)
            if mode == 0 and p.vec_bytes >= 4:
                chunks = (p.rows_per_tile * ng * R + 30) // 16
                assert p.smem_bytes == (16 * chunks + 127) // 128 * 128
            else:
                _, RS = region_stride(R, ng, p.rows_per_tile)
                assert p.smem_bytes == (ng * RS + 4 * ng + 15) // 16 * 16


def swz(x):
    return x ^ (((x >> 9) & 7) << 4)


def replay_gather_unit(R, ng, G, rows, S_tile, a_s, a_g):
    """Mode 0 with pieces of G >= 4 bytes: the segment's chunks at swizzled
    places of an image; threads build gathered chunks e = t + m*nthr0 of the
    regions laid end to end (Cpad chunks each), all of a thread's chunks
    sharing their phase within a run."""
    HDE = ng * R
    segB, L = rows * HDE, rows * R
    nS = (a_s + segB + 15) >> 4
    Cg = (S_tile * R + 30) // 16
    Rp = R // math.gcd(R, 16)
    nthr0 = Rp * (256 // Rp)
    Cpad = (Cg + Rp - 1) // Rp * Rp
    image = (16 * ((S_tile * HDE + 30) // 16) + 127) // 128 * 128
    r_n = (a_g + L + 15) >> 4
    rowsA = rows >> 1
    cI1 = (a_s + rowsA * HDE + 15) >> 4
    cB1 = (a_g + rowsA * R) >> 4
    # the image: chunk c at swz(16c), all inside the allocation
    places = {swz(16 * c) for c in range(nS)}
    assert len(places) == nS and max(places) + 16 <= image
    got = {}
    for tid in range(nthr0):
        q = 16 * tid - a_g + 16 * R
        col, drow, off = q % R, 0, []
        for _ in range(16 // G):
            off.append(drow * HDE + col)
            col += G
            if col == R:
                col, drow = 0, drow + 1
        for e in range(tid, ng * Cpad, nthr0):
            g, c = divmod(e, Cpad)
            if c >= r_n:
                continue
            q0 = 16 * c - a_g
            i0 = (q0 + 16 * R) // R - 16
            base = a_s + i0 * HDE + g * R
            for n in range(16 // G):
                qq = q0 + n * G
                if not 0 <= qq < L:
                    continue
                pos = base + off[n]                    # a_s + segment byte
                seg = pos - a_s
                i, cc = divmod(qq, R)
                assert seg == i * HDE + g * R + cc     # the element map
                assert 0 <= seg < segB and swz(pos) + G <= image
                if c < cB1:
                    assert (pos >> 4) < cI1, "built before its load batch landed"
                for b in range(G):
                    assert (g, qq + b) not in got
                    got[(g, qq + b)] = seg + b
    assert len(got) == ng * L


@pytest.mark.parametrize("R,G", [(12, 4), (20, 4), (36, 4), (8, 8), (24, 8), (200, 8), (4, 4), (40, 8)],
                         ids=lambda v: str(v))
def test_mode0_gather_placement(R, G):
    rng = random.Random(2000 + R)
    for ng in (1, 2, 3, 4, 8, 16, 27):
        if phase_movers(ng * R) < 128:
            continue
        for _ in range(3):
            S_tile = rng.choice([1, 2, 3, 64, max(1, 32768 // (ng * R))])
            rows = rng.randint(1, S_tile)
            replay_gather_unit(R, ng, G, rows, S_tile, rng.randrange(0, 16, G), rng.randrange(0, 16, G))
