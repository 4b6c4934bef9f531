"""The re-aligning (staged) copy path vs the CPU oracle, bit for bit (needs a B200).

The staged path takes the shapes whose runs ((H/w)*D*E bytes), row pitch or
slab base addresses are not 16-byte aligned: it moves every byte with aligned
16-byte global accesses and re-aligns them in shared memory in pieces of the
widest width those alignments allow. These tests run it (chosen by AUTO, or
forced) on narrow runs, misaligned bases, odd pitches, head-packed tensors,
chunked and windowed launches, the host-buffer entry point and a CUDA graph,
plus the vector-path benchmark shapes at full size; every output byte is
compared with the oracle and the bytes around each output slab must survive.
"""

import random

import pytest
import torch

import oracle
from sequence_all_re_b200 import PATH_AUTO, PATH_STAGED, PATH_VEC, UlyssesA2A
from synth import normal_slabs, random_byte_slabs, slab_shape, uniform_slabs
from test_parity_gpu import Guarded, bits, run_case

pytestmark = pytest.mark.gpu

INT = {1: torch.uint8, 2: torch.int16, 4: torch.int32, 8: torch.int64}

NARROW = [
    # (w, B, S_local, H, D, E): runs of (H/w)*D*E bytes, not a multiple of 16
    (4, 2, 100, 4, 3, 2),       # 6-byte runs: 2-byte pieces
    (4, 1, 77, 4, 3, 4),        # 12-byte runs: 4-byte pieces
    (8, 2, 53, 8, 100, 2),      # 200-byte runs: 8-byte pieces
    (3, 2, 29, 6, 5, 1),        # 10-byte runs: 2-byte pieces, odd rank count
    (2, 3, 33, 2, 7, 1),        # 7-byte runs: 1-byte pieces
    (2, 2, 40, 2, 1, 8),        # 8-byte runs (AUTO: the fixed-phase form, 8-byte pieces)
    (16, 1, 21, 16, 3, 2),      # w = 16
    (1, 2, 31, 3, 5, 2),        # w = 1: a copy
    (5, 1, 4000, 5, 3, 2),      # many rows per unit
]


@pytest.mark.parametrize("case", NARROW, ids=lambda c: "w{}B{}S{}H{}D{}E{}".format(*c))
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("chunked", [False, True], ids=["whole", "per_plane"])
def test_narrow_runs_take_the_staged_path(case, mode, chunked):
    # AUTO re-aligns pieces of 4 bytes or less through shared memory, and
    # 8-byte ones where the fixed-phase form applies; the staged path forced
    # gives the same bytes
    w, B, S, H, D, E = case
    shape = slab_shape(mode, w, B, S, H, D)
    xs = [t.view(INT[E]).reshape(shape)
          for t in random_byte_slabs(shape[:-1] + (shape[-1] * E,), w, seed0=100 + w + D)]
    with UlyssesA2A(0, E) as a2a:
        p = a2a.plan([t.cuda() for t in xs], mode)
        assert p["vec_bytes"] < 16
        # (8-byte pieces too: the fixed-phase form applies to every case here)
        assert p["path"] == PATH_STAGED
        run_case(xs, mode, chunked=chunked, a2a=a2a)
        run_case(xs, mode, chunked=chunked, a2a=a2a, path=PATH_STAGED)
        # dense rows and aligned slabs: the fixed-phase form, unless the
        # per-piece form is asked for
        assert a2a.plan([t.cuda() for t in xs], mode)["fixed_phase"] == 1
        run_case(xs, mode, chunked=chunked, a2a=a2a, path=PATH_STAGED, tuning=dict(staged_form=1))
        assert a2a.plan([t.cuda() for t in xs], mode)["fixed_phase"] == 0


SHAPES = [
    (2, 1, 64, 4, 64),
    (4, 2, 100, 8, 128),
    (8, 2, 53, 40, 128),
    (3, 2, 29, 6, 32),
    (1, 2, 33, 4, 64),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "w{}B{}S{}H{}D{}".format(*s))
@pytest.mark.parametrize("mode", [0, 1])
def test_forced_staged_on_aligned_shapes(shape, mode):
    # every alignment allows 16-byte pieces: the staged kernel's G = 16 form
    w, B, S, H, D = shape
    xs = normal_slabs(slab_shape(mode, w, B, S, H, D), w, "bf16", seed0=200 + S)
    for chunked in (False, True):
        for knobs in ({}, dict(rows_per_tile=1), dict(rows_per_tile=7), dict(ctas_per_sm=3)):
            run_case(xs, mode, chunked=chunked, path=PATH_STAGED, tuning=knobs)


@pytest.mark.parametrize("offset", [2, 4, 8, 6, 10, 14])
@pytest.mark.parametrize("side", ["in", "out"])
def test_misaligned_bases_every_offset(offset, side):
    w, B, S, H, D = 4, 2, 45, 8, 64
    xs = normal_slabs((B, S, H, D), w, "bf16", seed0=300 + offset)
    ys = oracle.ulysses_a2a(xs, 0)
    kw = {"in_offset": offset} if side == "in" else {"out_offset": offset}
    for mode, src in ((0, xs), (1, ys)):
        for chunked in (False, True):
            run_case(src, mode, chunked=chunked, **kw)


class _GuardedAt:
    """Output slabs at per-slab byte offsets past a 16-byte boundary, poisoned,
    with 64 guard bytes on either side."""

    def __init__(self, shape, dtype, offsets):
        self.nbytes = torch.empty(shape, dtype=dtype, device="meta").numel() * \
            torch.empty((), dtype=dtype).element_size()
        self.offsets = list(offsets)
        self.bufs, self.slabs = [], []
        for off in offsets:
            lo = 64 + off
            buf = torch.full((self.nbytes + 128 + 16,), 0x5A, dtype=torch.uint8, device="cuda")
            buf[lo:lo + self.nbytes].fill_(0xFF)
            self.bufs.append(buf)
            self.slabs.append(buf[lo:lo + self.nbytes].view(dtype).view(shape))

    def check_guards(self):
        for buf, off in zip(self.bufs, self.offsets):
            lo = 64 + off
            assert bool((buf[:lo] == 0x5A).all()), "bytes before an output slab were written"
            assert bool((buf[lo + self.nbytes:] == 0x5A).all()), "bytes after an output slab were written"


def _at(t, off):
    raw = torch.empty(t.numel() * t.element_size() + off, dtype=torch.uint8, device="cuda")
    v = raw[off:].view(t.dtype).view(t.shape)
    v.copy_(t)
    return v


def _run_at(a2a, xs_cpu, mode, in_offs, out_offs, chunked, fixed_phase):
    """One call with slab k of the inputs in_offs[k] and of the outputs out_offs[k]
    bytes past a 16-byte boundary; the plan's form is checked, then every byte
    against the oracle and the bytes around the outputs."""
    w = len(xs_cpu)
    xs = [_at(t, o) for t, o in zip(xs_cpu, in_offs)]
    g = _GuardedAt(oracle.output_shape(tuple(xs_cpu[0].shape), mode, w), xs_cpu[0].dtype, out_offs)
    p = a2a.plan(xs, mode, out=g.slabs)
    assert p["path"] == PATH_STAGED and p["fixed_phase"] == fixed_phase, p
    a2a.run(xs, mode, chunked=chunked, out=g.slabs)
    a2a.status()
    want = oracle.ulysses_a2a(xs_cpu, mode)
    for k in range(w):
        assert torch.equal(bits(g.slabs[k].cpu()), bits(want[k])), k
    g.check_guards()


# (w, B, S_local, H, D, E): dense narrow runs of 6, 12, 5, 10, 20 and 36 bytes
PHASE = [(4, 2, 300, 4, 3, 2), (4, 1, 257, 4, 3, 4), (2, 2, 97, 2, 5, 1), (3, 2, 151, 3, 5, 2),
         (3, 1, 211, 6, 5, 2), (8, 1, 99, 8, 9, 4)]


@pytest.mark.parametrize("case", PHASE, ids=lambda c: "w{}B{}S{}H{}D{}E{}".format(*c))
@pytest.mark.parametrize("mode", [0, 1])
def test_fixed_phase_form_every_offset(case, mode):
    # the gathered slabs at one offset (every piece-aligned value), the strided
    # slabs each at its own: the fixed-phase kernel, whole and per plane
    w, B, S, H, D, E = case
    shape = slab_shape(mode, w, B, S, H, D)
    xs = [t.view(INT[E]).reshape(shape)
          for t in random_byte_slabs(shape[:-1] + (shape[-1] * E,), w, seed0=900 + S)]
    G = 1
    while G < 8 and ((H // w) * D * E) % (2 * G) == 0:
        G *= 2
    with UlyssesA2A(0, E) as a2a:
        for a in range(0, 16, G):
            strided = [(a + 3 * G * k) % 16 for k in range(w)]
            gathered = [a] * w
            ins, outs = (strided, gathered) if mode == 0 else (gathered, strided)
            for chunked in (False, True):
                _run_at(a2a, xs, mode, ins, outs, chunked, 1)


@pytest.mark.parametrize("mode", [0, 1])
def test_per_piece_form_when_gathered_offsets_differ(mode):
    w, B, S, H, D, E = 4, 2, 300, 4, 3, 2
    shape = slab_shape(mode, w, B, S, H, D)
    xs = [t.view(torch.int16).reshape(shape)
          for t in random_byte_slabs(shape[:-1] + (shape[-1] * E,), w, seed0=950)]
    with UlyssesA2A(0, E) as a2a:
        gathered, strided = [0, 2, 4, 6], [2] * w
        ins, outs = (strided, gathered) if mode == 0 else (gathered, strided)
        _run_at(a2a, xs, mode, ins, outs, False, 0)


@pytest.mark.parametrize("mode", [0, 1])
def test_fixed_phase_form_with_few_rows_per_unit(mode):
    # units of 1, 2 and 5 rows (24 to 120 strided bytes): most threads move no
    # strided chunk, and a unit's first and last chunks are partial
    w, B, S, H, D, E = 4, 2, 37, 4, 3, 2
    shape = slab_shape(mode, w, B, S, H, D)
    xs = [t.view(torch.int16).reshape(shape)
          for t in random_byte_slabs(shape[:-1] + (shape[-1] * E,), w, seed0=960)]
    with UlyssesA2A(0, E) as a2a:
        for rows in (1, 2, 5):
            a2a.set_tuning(rows_per_tile=rows)
            _run_at(a2a, xs, mode, [2] * w, [6] * w, False, 1)
            _run_at(a2a, xs, mode, [0] * w, [0] * w, True, 1)


def test_pitched_slabs_through_the_staged_path():
    # q, k, v read in place from a packed projection output whose row is
    # 3*H*D + 4 elements (8-byte aligned rows), and mode 1 back into it: the
    # gap elements are never touched
    w, B, S, H, D = 4, 2, 37, 8, 16
    pitch = 3 * H * D + 4
    bufs_cpu = normal_slabs((B * S * pitch,), w, "bf16", seed0=400)
    with UlyssesA2A(0, 2) as a2a:
        a2a.set_path(PATH_STAGED)                 # 8-byte pieces: AUTO would take VEC
        bufs = [t.cuda() for t in bufs_cpu]
        for c in range(3):
            views = [t[c * H * D:].as_strided((B, S, H, D), (S * pitch, pitch, D, 1)) for t in bufs]
            p = a2a.plan(views, 0)
            assert p["path"] == PATH_STAGED and p["row_pitch"] == pitch
            want = oracle.ulysses_a2a_pitched(bufs_cpu, 0, w, B, S, H, D, pitch, offset=c * H * D)
            for chunked in (False, True):
                out = a2a.run(views, 0, chunked=chunked)
                for r in range(w):
                    assert torch.equal(bits(out[r].cpu()).reshape(-1), bits(want[r])), (c, r)
            dst = [torch.full_like(t, float("nan")) for t in bufs]
            dviews = [t[c * H * D:].as_strided((B, S, H, D), (S * pitch, pitch, D, 1)) for t in dst]
            a2a.run(out, 1, out=dviews)
            a2a.status()
            for j in range(w):
                got = dst[j].cpu().view(B * S, pitch)
                src = bufs_cpu[j].view(B * S, pitch)
                lo, hi = c * H * D, (c + 1) * H * D
                assert torch.equal(bits(got[:, lo:hi].contiguous()), bits(src[:, lo:hi].contiguous()))
                rest = torch.cat([got[:, :lo], got[:, hi:]], dim=1)
                assert bool(torch.isnan(rest.float()).all()), "a gap or another slot was written"


@pytest.mark.parametrize("T", [2, 3])
def test_packed_tensors_through_the_staged_path(T):
    # D = 13: 26-byte runs, 2-byte pieces; one launch for all T tensors
    w, B, S, H, D = 4, 2, 41, 8, 13
    packed_cpu = normal_slabs((B, S, T, H, D), w, "bf16", seed0=500 + T)
    flat = [t.reshape(-1) for t in packed_cpu]
    with UlyssesA2A(0, 2) as a2a:
        packed = [t.cuda() for t in packed_cpu]
        for chunked in (False, True):
            n0 = a2a.launch_count
            outs = a2a.run_packed(packed, 0, chunked=chunked)
            assert a2a.launch_count - n0 == (B if chunked else 1)
            for t in range(T):
                want = oracle.ulysses_a2a_pitched(flat, 0, w, B, S, H, D, T * H * D,
                                                  offset=t * H * D)
                for r in range(w):
                    assert torch.equal(bits(outs[t][r].cpu()).reshape(-1), bits(want[r])), (t, r)
            back = [torch.full((B, S, T, H, D), -1, dtype=torch.int16, device="cuda")
                    .view(torch.bfloat16) for _ in range(w)]
            a2a.run_packed(outs, 1, chunked=chunked, out=back)
            a2a.status()
            for j in range(w):
                assert torch.equal(bits(back[j].cpu()), bits(packed_cpu[j])), j


def test_windowed_and_host_buffer_variants():
    w, B, S, H, D = 4, 3, 50, 4, 3
    xs = normal_slabs((B, S, H, D), w, "bf16", seed0=600)
    want = oracle.ulysses_a2a(xs, 0)
    with UlyssesA2A(0, 2) as a2a:
        out = a2a.run([t.cuda() for t in xs], 0, chunked=2)
        a2a.status()
        for r in range(w):
            assert torch.equal(bits(out[r].cpu()), bits(want[r]))
        host_out = a2a.run_host([t.pin_memory() for t in xs], 0)
        for r in range(w):
            assert torch.equal(bits(host_out[r]), bits(want[r]))
        back = a2a.run_host(host_out, 1)
        for j in range(w):
            assert torch.equal(bits(back[j]), bits(xs[j]))


def test_staged_launch_captures_into_a_cuda_graph():
    w, B, S, H, D = 4, 2, 64, 4, 3
    xs = normal_slabs((B, S, H, D), w, "bf16", seed0=650)
    want = oracle.ulysses_a2a(xs, 0)
    with UlyssesA2A(0, 2) as a2a:
        xd = [t.cuda() for t in xs]
        out = [torch.empty(B, S * w, H // w, D, dtype=torch.bfloat16, device="cuda")
               for _ in range(w)]
        stream = torch.cuda.Stream()
        with torch.cuda.stream(stream):
            a2a.run(xd, 0, out=out, stream=stream)       # first call sets the kernel attributes
        torch.cuda.synchronize()
        for o in out:
            o.view(torch.int16).fill_(-1)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            a2a.run(xd, 0, out=out, stream=stream)
        g.replay()
        torch.cuda.synchronize()
        for r in range(w):
            assert torch.equal(bits(out[r].cpu()), bits(want[r]))


def test_randomized_staged_cases():
    """80 seeded random cases on the staged path: rank counts 1..16, ragged
    S_local, odd D, element sizes 1/2/4/8, random base offsets on both sides,
    row pitches, head-packed tensors, both modes, chunked 0/1, random rows per
    unit; compared with the (pitched) oracle and the guard bands checked."""
    rng = random.Random(77001)
    ctxs = {E: UlyssesA2A(0, E) for E in (1, 2, 4, 8)}
    try:
        for case in range(80):
            E = rng.choice([1, 2, 4, 8])
            w = rng.choice([1, 2, 3, 4, 5, 8, 16])
            T = rng.choice([1, 1, 1, 2, 3]) if w <= 16 else 1
            Hw = rng.randint(1, 3)
            H, B, S = Hw * w, rng.randint(1, 3), rng.randint(1, 90)
            D = rng.choice([1, 3, 5, 8, 13, 24, 64, 100])
            if T * H * D * E > 64 * 1024:
                D = 3
            mode, chunked = rng.randint(0, 1), rng.randint(0, 1)
            a2a = ctxs[E]
            a2a.set_path(rng.choice([PATH_AUTO, PATH_STAGED]))
            a2a.set_tuning(rows_per_tile=rng.choice([0, 0, 1, 3, 17]))
            dt = INT[E]
            seed = 70000 + case
            if T == 1:
                pitch = H * D + rng.choice([0, 0, 1, 2, 8])
                off_in = rng.choice([0, 0, E, 2 * E, 4 * E]) % 16
                off_out = rng.choice([0, 0, E, 8]) % 16
                off_out -= off_out % E
                n_p = (B * S - 1) * pitch + H * D
                n_d = B * S * H * D
                if mode == 0:
                    bufs = [t.view(dt) for t in random_byte_slabs((n_p * E,), w, seed0=seed)]
                    want = oracle.ulysses_a2a_pitched(bufs, 0, w, B, S, H, D, pitch)
                    dev = []
                    for t in bufs:
                        raw = torch.empty(n_p * E + off_in, dtype=torch.uint8, device="cuda")
                        v = raw[off_in:].view(dt)
                        v.copy_(t)
                        dev.append(v.as_strided((B, S, H, D), (S * pitch, pitch, D, 1)))
                    g = Guarded((B, S * w, H // w, D), dt, w, offset=off_out)
                    a2a.run(dev, 0, chunked=bool(chunked), out=g.slabs)
                    a2a.status()
                    for r in range(w):
                        assert torch.equal(g.slabs[r].cpu().reshape(-1), want[r]), (case, r)
                    g.check_guards()
                else:
                    ins = [t.view(dt) for t in random_byte_slabs((n_d * E,), w, seed0=seed)]
                    poison = [torch.full((n_p * E,), 0xA5, dtype=torch.uint8).view(dt)
                              for _ in range(w)]
                    want = oracle.ulysses_a2a_pitched(ins, 1, w, B, S, H, D, pitch,
                                                      out_bufs=[p.clone() for p in poison])
                    xs = []
                    for t in ins:
                        raw = torch.empty(n_d * E + off_in, dtype=torch.uint8, device="cuda")
                        v = raw[off_in:].view(dt)
                        v.copy_(t)
                        xs.append(v.view(B, S * w, H // w, D))
                    dst = []
                    for p_ in poison:
                        raw = torch.empty(n_p * E + off_out, dtype=torch.uint8, device="cuda")
                        v = raw[off_out:].view(dt)
                        v.copy_(p_)
                        dst.append(v)
                    out = [t.as_strided((B, S, H, D), (S * pitch, pitch, D, 1)) for t in dst]
                    a2a.run(xs, 1, chunked=bool(chunked), out=out)
                    a2a.status()
                    for j in range(w):
                        assert torch.equal(dst[j].cpu(), want[j].reshape(-1)), (case, j)
            else:
                packed_cpu = [t.view(dt).reshape(B, S, T, H, D)
                              for t in random_byte_slabs((B, S, T, H, D * E), w, seed0=seed)]
                packed = [t.cuda() for t in packed_cpu]
                outs = a2a.run_packed(packed, 0, chunked=bool(chunked))
                flat = [t.reshape(-1) for t in packed_cpu]
                for t in range(T):
                    want = oracle.ulysses_a2a_pitched(flat, 0, w, B, S, H, D, T * H * D,
                                                      offset=t * H * D)
                    for r in range(w):
                        assert torch.equal(outs[t][r].cpu().reshape(-1), want[r]), (case, t, r)
                back = a2a.run_packed(outs, 1, chunked=not chunked)
                a2a.status()
                for j in range(w):
                    assert torch.equal(back[j].cpu(), packed_cpu[j]), (case, j)
    finally:
        for c in ctxs.values():
            c.close()


# the vector-path benchmark shapes at full size: (w, B, S, H, D, E, base offset)
FULL_VEC = {
    "rows200B_w8_S41943_H8_D100": (8, 1, 41943, 8, 100, 2, 0),
    "rows12B_w4_S1398101_H4_D3_fp32": (4, 1, 1398101, 4, 3, 4, 0),
    "rows6B_w4_S2796202_H4_D3": (4, 1, 2796202, 4, 3, 2, 0),
    "base8_w4_S8192_H24_D128": (4, 1, 8192, 24, 128, 2, 8),
    "base2_w4_S8192_H24_D128": (4, 1, 8192, 24, 128, 2, 2),
}


@pytest.mark.parametrize("name", sorted(FULL_VEC))
def test_vector_path_benchmark_shapes_full_size(name):
    w, B, S, H, D, E, off = FULL_VEC[name]
    make = normal_slabs if E == 2 else uniform_slabs
    xs = make((B, S, H, D), w, "bf16" if E == 2 else "fp32", seed0=800)
    ys = run_case(xs, 0, in_offset=off, out_offset=off)     # compared with the oracle inside
    run_case(ys, 1, in_offset=off, out_offset=off)
