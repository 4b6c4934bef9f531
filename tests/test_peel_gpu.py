"""The vector kernel's peeled form vs the CPU oracle, bit for bit (needs a B200).

When every slab starts the same number of bytes a past a 16-byte boundary and
runs and rows are whole multiples of 16 bytes, the vector kernel moves each
run's 16-byte vectors between a head of 16 - a bytes and a tail of a bytes,
which its first CTAs move in aligned pieces. The re-layout is the
one the FastVideo API docs give for ``run_armed`` (device_communicators/
ulysses_a2a): out_r[b, j*S_local + s, h', d] = x_j[b, s, r*(H/w) + h', d] in
mode 0, its inverse in mode 1. Every output slab here is poisoned and fenced
by canary bytes (``Guarded``), so a byte the kernel skips or writes past a
slab's end fails the comparison.
"""

import random

import pytest
import torch

import oracle
from sequence_all_re_b200 import PATH_AUTO, PATH_VEC, UlyssesA2A, _lib
from synth import normal_slabs, random_byte_slabs, slab_shape
from test_parity_gpu import Guarded, bits

pytestmark = pytest.mark.gpu

INT = {1: torch.uint8, 2: torch.int16, 4: torch.int32, 8: torch.int64}


def _offset_slabs(cpu, offset):
    """Device copies of the CPU slabs, each `offset` bytes past a 256-byte boundary."""
    out = []
    for t in cpu:
        n = t.numel() * t.element_size()
        raw = torch.empty(n + offset, dtype=torch.uint8, device="cuda")
        v = raw[offset:].view(t.dtype).view(t.shape)
        v.copy_(t)
        out.append(v)
    return out


def _check(a2a, xs_cpu, mode, offset, chunked, expect_peeled=True, out_offset=None):
    """Inputs `offset` bytes past a boundary, outputs `out_offset` (default: the
    same); the plan must be the peeled form expected (1 = one offset, 2 = two)."""
    w = len(xs_cpu)
    xs = _offset_slabs(xs_cpu, offset)
    oshape = oracle.output_shape(tuple(xs_cpu[0].shape), mode, w)
    g = Guarded(oshape, xs_cpu[0].dtype, w, offset=offset if out_offset is None else out_offset)
    p = a2a.plan(xs, mode, chunked=chunked, out=g.slabs)
    assert p["path"] == PATH_VEC and p["peeled"] == int(expect_peeled), p
    a2a.run(xs, mode, chunked=chunked, out=g.slabs)
    a2a.status()
    want = oracle.ulysses_a2a(xs_cpu, mode)
    for k in range(w):
        assert torch.equal(bits(g.slabs[k].cpu()), bits(want[k])), f"rank {k}"
    g.check_guards()
    return [s.cpu() for s in g.slabs]


CASES = [
    # (w, B, S_local, H, D, E): runs of (H/w)*D*E bytes
    (4, 2, 45, 8, 64, 2),        # 256-byte runs
    (8, 2, 53, 40, 128, 2),      # the ragged-tail workload's heads, short sequence
    (2, 3, 17, 4, 40, 2),        # 80-byte runs
    (4, 1, 13, 8, 32, 4),        # fp32, 256-byte runs
    (2, 2, 11, 4, 40, 1),        # 1-byte elements: odd offsets
    (2, 2, 19, 2, 8, 8),         # 8-byte elements, 64-byte runs (the shortest peeled)
    (1, 2, 9, 4, 40, 2),         # w = 1: a copy, 320-byte runs
    (16, 1, 21, 16, 64, 2),      # w = 16
    (3, 2, 29, 6, 32, 2),        # odd rank count
]


def _offsets(E):
    return [o for o in range(E, 16, E)] if E < 8 else [8]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "w{}B{}S{}H{}D{}E{}".format(*c))
@pytest.mark.parametrize("mode", [0, 1])
def test_slabs_at_one_offset_every_offset(case, mode):
    w, B, S, H, D, E = case
    shape = slab_shape(mode, w, B, S, H, D)
    xs = [t.view(INT[E]).reshape(shape)
          for t in random_byte_slabs(shape[:-1] + (shape[-1] * E,), w, seed0=700 + w + D)]
    with UlyssesA2A(0, E) as a2a:
        for off in _offsets(E):
            for chunked in (False, True):
                _check(a2a, xs, mode, off, chunked)
        # the vector path forced takes the same windows; so does a grid-stride
        # grid of one CTA per SM over one-row units
        a2a.set_path(PATH_VEC)
        _check(a2a, xs, mode, _offsets(E)[0], False)
        a2a.set_tuning(ctas_per_sm=1, rows_per_tile=1)
        _check(a2a, xs, mode, _offsets(E)[-1], True)
        _check(a2a, xs, mode, _offsets(E)[0], False, expect_peeled=2, out_offset=0)


@pytest.mark.parametrize("E", [1, 2, 4, 8])
@pytest.mark.parametrize("mode", [0, 1])
def test_inputs_and_outputs_at_two_offsets(E, mode):
    # every pair of different offsets (multiples of E) on the two sides: each
    # destination vector, head and tail is joined from two aligned source
    # vectors (peeled = 2)
    w, B, S, H, D = 4, 2, 29, 8, 128 // E
    shape = slab_shape(mode, w, B, S, H, D)
    xs = [t.view(INT[E]).reshape(shape)
          for t in random_byte_slabs(shape[:-1] + (shape[-1] * E,), w, seed0=770 + E + mode)]
    offs = list(range(0, 16, E))
    with UlyssesA2A(0, E) as a2a:
        for a_in in offs:
            for a_out in offs:
                if a_in != a_out:
                    _check(a2a, xs, mode, a_in, (a_in + a_out) % 2 == 0, expect_peeled=2,
                           out_offset=a_out)


@pytest.mark.parametrize("mode", [0, 1])
def test_offset_slabs_through_the_staging_window(mode):
    # chunked = 2 copies every plane into the context's (aligned) window and
    # re-lays it out from there into the caller's slabs, 6 bytes off: the
    # shifted kernel in mode 0 (aligned window -> offset outputs); in mode 1
    # the window holds the gathered plane and the outputs are offset too
    w, B, S, H, D = 4, 3, 45, 8, 64
    shape = slab_shape(mode, w, B, S, H, D)
    xs_cpu = normal_slabs(shape, w, "bf16", seed0=785 + mode)
    with UlyssesA2A(0, 2) as a2a:
        xs = _offset_slabs(xs_cpu, 6)
        oshape = oracle.output_shape(shape, mode, w)
        g = Guarded(oshape, torch.bfloat16, w, offset=6)
        n0 = a2a.launch_count
        a2a.run(xs, mode, chunked=2, out=g.slabs)
        a2a.status()
        assert a2a.launch_count - n0 == B
        want = oracle.ulysses_a2a(xs_cpu, mode)
        for k in range(w):
            assert torch.equal(bits(g.slabs[k].cpu()), bits(want[k])), k
        g.check_guards()


def test_shifted_round_trip_chunked_and_pitched():
    # inputs 2 bytes off, outputs 10 off, chunked per plane; then mode 1 from
    # aligned slabs into q slots of a packed buffer 6 bytes off
    w, B, S, H, D = 4, 3, 100, 8, 128
    xs = normal_slabs((B, S, H, D), w, "bf16", seed0=780)
    with UlyssesA2A(0, 2) as a2a:
        ys = _check(a2a, xs, 0, 2, True, expect_peeled=2, out_offset=10)
        pitch = 3 * H * D
        bufs = _offset_slabs([torch.full((B * S * pitch,), float("nan"), dtype=torch.bfloat16)
                              for _ in range(w)], 6)
        views = [t.as_strided((B, S, H, D), (S * pitch, pitch, D, 1)) for t in bufs]
        dense = [y.cuda() for y in ys]
        p = a2a.plan(dense, 1, out=views)
        assert p["peeled"] == 2 and p["row_pitch"] == pitch
        a2a.run(dense, 1, out=views)
        a2a.status()
        for j in range(w):
            got = bufs[j].cpu().view(B * S, pitch)
            assert torch.equal(bits(got[:, :H * D].contiguous()), bits(xs[j].reshape(B * S, H * D)))
            assert bool(torch.isnan(got[:, H * D:].float()).all()), "another slot was written"


def test_shifted_packed_tensors():
    w, B, S, H, D, T = 4, 2, 41, 8, 64, 3
    packed_cpu = normal_slabs((B, S, T, H, D), w, "bf16", seed0=790)
    flat = [t.reshape(-1) for t in packed_cpu]
    with UlyssesA2A(0, 2) as a2a:
        packed = _offset_slabs(packed_cpu, 14)
        outs = [[_offset_slabs([torch.empty(B, S * w, H // w, D, dtype=torch.bfloat16)], 4)[0]
                 for _ in range(w)] for _ in range(T)]
        flat_out = [o.data_ptr() for per_t in outs for o in per_t]
        rc, p, msg = _lib.ulysses_a2a_plan_ex([t.data_ptr() for t in packed], flat_out, B, S, H, D,
                                              w, 0, 0, 2, ntensors=T)
        assert rc == _lib.OK and p.peeled == 2, msg
        a2a.run_packed(packed, 0, out=outs)
        a2a.status()
        for t in range(T):
            want = oracle.ulysses_a2a_pitched(flat, 0, w, B, S, H, D, T * H * D, offset=t * H * D)
            for r in range(w):
                assert torch.equal(bits(outs[t][r].cpu()).reshape(-1), bits(want[r])), (t, r)


def test_round_trip_through_peeled_launches():
    w, B, S, H, D = 4, 3, 100, 8, 128
    xs = normal_slabs((B, S, H, D), w, "bf16", seed0=710)
    with UlyssesA2A(0, 2) as a2a:
        ys = _check(a2a, xs, 0, 6, False)
        back = _check(a2a, ys, 1, 6, True)
        for j in range(w):
            assert torch.equal(bits(back[j]), bits(xs[j]))


def test_offsets_that_differ_between_slabs_are_not_peeled():
    # one output slab 2 bytes further off: the offsets no longer match and AUTO
    # re-aligns in shared memory instead (same bytes)
    w, B, S, H, D = 4, 2, 33, 8, 64
    xs_cpu = normal_slabs((B, S, H, D), w, "bf16", seed0=720)
    with UlyssesA2A(0, 2) as a2a:
        xs = _offset_slabs(xs_cpu, 2)
        g = Guarded((B, S * w, H // w, D), torch.bfloat16, w, offset=2)
        odd = Guarded((B, S * w, H // w, D), torch.bfloat16, 1, offset=4)
        outs = g.slabs[:-1] + odd.slabs
        p = a2a.plan(xs, 0, out=outs)
        assert p["peeled"] == 0 and p["path"] != PATH_VEC
        a2a.run(xs, 0, out=outs)
        a2a.status()
        want = oracle.ulysses_a2a(xs_cpu, 0)
        for k in range(w):
            assert torch.equal(bits(outs[k].cpu()), bits(want[k]))
        g.check_guards()
        odd.check_guards()


def test_pitched_views_of_a_packed_buffer():
    # q, k and v of a packed [B, S, 3, H, D] buffer that starts 6 bytes past a
    # boundary, the dense side 6 bytes past too: both modes peel; mode 1 writes
    # back into the packed slots and leaves the other slots untouched
    w, B, S, H, D = 4, 2, 37, 8, 64
    pitch = 3 * H * D
    off = 6
    bufs_cpu = normal_slabs((B * S * pitch,), w, "bf16", seed0=730)
    with UlyssesA2A(0, 2) as a2a:
        bufs = _offset_slabs(bufs_cpu, off)
        for c in range(3):
            views = [t[c * H * D:].as_strided((B, S, H, D), (S * pitch, pitch, D, 1)) for t in bufs]
            g = Guarded((B, S * w, H // w, D), torch.bfloat16, w, offset=off)
            p = a2a.plan(views, 0, out=g.slabs)
            assert p["peeled"] == 1 and p["row_pitch"] == pitch
            want = oracle.ulysses_a2a_pitched(bufs_cpu, 0, w, B, S, H, D, pitch, offset=c * H * D)
            for chunked in (False, True):
                a2a.run(views, 0, chunked=chunked, out=g.slabs)
                a2a.status()
                for r in range(w):
                    assert torch.equal(bits(g.slabs[r].cpu()).reshape(-1), bits(want[r])), (c, r)
                g.check_guards()
            dst = _offset_slabs([torch.full_like(t, float("nan")) for t in bufs_cpu], off)
            dviews = [t[c * H * D:].as_strided((B, S, H, D), (S * pitch, pitch, D, 1)) for t in dst]
            p = a2a.plan(g.slabs, 1, out=dviews)
            assert p["peeled"] == 1
            a2a.run(g.slabs, 1, out=dviews)
            a2a.status()
            for j in range(w):
                got = dst[j].cpu().view(B * S, pitch)
                src = bufs_cpu[j].view(B * S, pitch)
                lo, hi = c * H * D, (c + 1) * H * D
                assert torch.equal(bits(got[:, lo:hi].contiguous()), bits(src[:, lo:hi].contiguous()))
                rest = torch.cat([got[:, :lo], got[:, hi:]], dim=1)
                assert bool(torch.isnan(rest.float()).all()), "a gap or another slot was written"


@pytest.mark.parametrize("T", [2, 3])
def test_packed_tensors_with_a_shared_offset(T):
    w, B, S, H, D = 4, 2, 41, 8, 64
    off = 10
    packed_cpu = normal_slabs((B, S, T, H, D), w, "bf16", seed0=740 + T)
    flat = [t.reshape(-1) for t in packed_cpu]
    with UlyssesA2A(0, 2) as a2a:
        packed = _offset_slabs(packed_cpu, off)
        outs = [[_offset_slabs([torch.empty(B, S * w, H // w, D, dtype=torch.bfloat16)], off)[0]
                 for _ in range(w)] for _ in range(T)]
        flat_out = [o.data_ptr() for per_t in outs for o in per_t]
        rc, p, msg = _lib.ulysses_a2a_plan_ex([t.data_ptr() for t in packed], flat_out, B, S, H, D,
                                              w, 0, 0, 2, ntensors=T)
        assert rc == _lib.OK and p.path == PATH_VEC and p.peeled == 1, msg
        for chunked in (False, True):
            n0 = a2a.launch_count
            a2a.run_packed(packed, 0, chunked=chunked, out=outs)
            assert a2a.launch_count - n0 == (B if chunked else 1)
            for t in range(T):
                want = oracle.ulysses_a2a_pitched(flat, 0, w, B, S, H, D, T * H * D,
                                                  offset=t * H * D)
                for r in range(w):
                    assert torch.equal(bits(outs[t][r].cpu()).reshape(-1), bits(want[r])), (t, r)
            back = _offset_slabs([torch.full((B, S, T, H, D), -1, dtype=torch.int16)
                                  .view(torch.bfloat16) for _ in range(w)], off)
            a2a.run_packed(outs, 1, chunked=chunked, out=back)
            a2a.status()
            for j in range(w):
                assert torch.equal(bits(back[j].cpu()), bits(packed_cpu[j])), j


def test_peeled_launch_captures_into_a_cuda_graph():
    w, B, S, H, D = 4, 2, 64, 8, 64
    xs_cpu = normal_slabs((B, S, H, D), w, "bf16", seed0=750)
    want = oracle.ulysses_a2a(xs_cpu, 0)
    with UlyssesA2A(0, 2) as a2a:
        xs = _offset_slabs(xs_cpu, 4)
        out = _offset_slabs([torch.empty(B, S * w, H // w, D, dtype=torch.bfloat16)
                             for _ in range(w)], 4)
        assert a2a.plan(xs, 0, out=out)["peeled"] == 1
        stream = torch.cuda.Stream()
        with torch.cuda.stream(stream):
            a2a.run(xs, 0, out=out, stream=stream)
        torch.cuda.synchronize()
        for o in out:
            o.view(torch.int16).fill_(-1)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            a2a.run(xs, 0, out=out, stream=stream)
        graph.replay()
        torch.cuda.synchronize()
        for r in range(w):
            assert torch.equal(bits(out[r].cpu()), bits(want[r]))


def test_randomized_shared_offset_cases():
    """60 seeded random cases: rank counts 1..16, ragged S_local, element sizes
    1/2/4/8, a random base offset for the inputs and, half the time, another
    for the outputs, random unit sizes; each checked against the oracle
    whichever path the planner takes, and the peeled form (1 for one offset,
    2 for two) required wherever its conditions hold (an offset, runs of 64
    bytes or more and a multiple of 16)."""
    rng = random.Random(760)
    n_peeled = 0
    ctxs = {}
    try:
        for case in range(60):
            E = rng.choice([1, 2, 2, 4, 8])
            w = rng.choice([1, 2, 3, 4, 8, 16])
            hw = rng.randint(1, 4)
            H = hw * w
            D = rng.choice([8, 16, 24, 32, 40, 64, 100, 128]) // (E if E > 2 else 1) or 1
            B, S = rng.randint(1, 3), rng.randint(1, 70)
            mode = rng.choice([0, 1])
            off = rng.randrange(0, 16, E) if E < 16 else 0
            off_out = off if rng.random() < 0.5 else rng.randrange(0, 16, E)
            shape = slab_shape(mode, w, B, S, H, D)
            xs = [t.view(INT[E]).reshape(shape)
                  for t in random_byte_slabs(shape[:-1] + (shape[-1] * E,), w, seed0=900 + case)]
            a2a = ctxs.setdefault(E, UlyssesA2A(0, E))
            a2a.set_path(PATH_AUTO)
            # unit sizes, both unit numberings, and grid-stride grids
            a2a.set_tuning(rows_per_tile=rng.choice([0, 0, 1, 5]), order=rng.choice([-1, 0, 1]),
                           ctas_per_sm=rng.choice([0, 0, 1, 3]))
            dev = _offset_slabs(xs, off)
            oshape = oracle.output_shape(shape, mode, w)
            g = Guarded(oshape, xs[0].dtype, w, offset=off_out)
            chunked = rng.choice([False, True])
            p = a2a.plan(dev, mode, chunked=chunked, out=g.slabs)
            run_bytes = hw * D * E
            if (off or off_out) and run_bytes >= 64 and run_bytes % 16 == 0:
                assert p["peeled"] == (1 if off == off_out else 2), (case, p)
            n_peeled += p["peeled"]
            a2a.run(dev, mode, chunked=chunked, out=g.slabs)
            a2a.status()
            want = oracle.ulysses_a2a(xs, mode)
            for k in range(w):
                assert torch.equal(bits(g.slabs[k].cpu()), bits(want[k])), (case, k)
            g.check_guards()
        assert n_peeled >= 10
    finally:
        for c in ctxs.values():
            c.close()
