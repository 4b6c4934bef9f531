"""CUDA path vs the CPU oracle, bit for bit (needs a B200).

Every output slab sits inside a larger buffer: the slab itself is pre-filled
with 0xFF (an element the kernel never writes stays wrong) and the bytes before
and after it hold a canary pattern that must survive the run (a write past
either end of a slab is caught). Inputs come from ``synth`` with fixed seeds;
expected values come from ``oracle`` only.
"""

import pytest
import torch

import oracle
from sequence_all_re_b200 import (A2AError, PATH_AUTO, PATH_STAGED, PATH_TMA, PATH_VEC, UlyssesA2A,
                                  _lib)
from synth import (normal_slabs, random_byte_slabs, rank_tagged_slabs, slab_shape, uniform_slabs,
                   unique_slabs)

pytestmark = pytest.mark.gpu

GUARD = 4096          # canary bytes on each side of an output slab (keeps 256 B alignment)
CANARY = 0xA5

INT_OF = {1: torch.uint8, 2: torch.int16, 4: torch.int32, 8: torch.int64}


def bits(t):
    return t.contiguous().view(INT_OF[t.element_size()])


class Guarded:
    """w output slabs, each poisoned and surrounded by canary bytes."""

    def __init__(self, shape, dtype, w, device="cuda", offset=0):
        n = 1
        for v in shape:
            n *= v
        esz = torch.empty((), dtype=dtype).element_size()
        self.nbytes = n * esz
        self.offset = offset
        self.bufs, self.slabs = [], []
        for _ in range(w):
            buf = torch.full((self.nbytes + 2 * GUARD + offset,), CANARY, dtype=torch.uint8,
                             device=device)
            lo = GUARD + offset
            buf[lo:lo + self.nbytes].fill_(0xFF)
            self.bufs.append(buf)
            self.slabs.append(buf[lo:lo + self.nbytes].view(dtype).view(shape))

    def check_guards(self):
        for buf in self.bufs:
            lo = GUARD + self.offset
            head = buf[:lo]
            tail = buf[lo + self.nbytes:]
            assert bool((head == CANARY).all()), "bytes before an output slab were written"
            assert bool((tail == CANARY).all()), "bytes after an output slab were written"


def run_case(xs_cpu, mode, *, chunked=False, path=PATH_AUTO, tuning=None, a2a=None,
             out_offset=0, in_offset=0):
    """Run the GPU path on xs_cpu (moved to the device) and compare with the oracle."""
    w = len(xs_cpu)
    E = xs_cpu[0].element_size()
    own = a2a is None
    a2a = a2a or UlyssesA2A(0, E)
    try:
        a2a.set_path(path)
        a2a.set_tuning(**(tuning or {}))
        if in_offset:
            xs = []
            for t in xs_cpu:
                raw = torch.empty(t.numel() * E + in_offset, dtype=torch.uint8, device="cuda")
                v = raw[in_offset:].view(t.dtype).view(t.shape)
                v.copy_(t)
                xs.append(v)
        else:
            xs = [t.cuda() for t in xs_cpu]
        oshape = oracle.output_shape(tuple(xs_cpu[0].shape), mode, w)
        g = Guarded(oshape, xs_cpu[0].dtype, w, offset=out_offset)
        before = a2a.launch_count
        a2a.run(xs, mode, chunked=chunked, out=g.slabs)
        a2a.status()
        B = xs_cpu[0].shape[0]
        assert a2a.launch_count - before == (B if chunked else 1)
        want = oracle.ulysses_a2a(xs_cpu, mode, chunked=False)
        for k in range(w):
            got = g.slabs[k].cpu()
            assert torch.equal(bits(got), bits(want[k])), f"rank {k} differs from the oracle"
        g.check_guards()
        return [s.cpu() for s in g.slabs]
    finally:
        if own:
            a2a.close()


# ---- small and medium shapes: several tiles, ragged tails, both paths -------

SHAPES = [
    # (w, B, S_local, H, D)
    (2, 1, 64, 4, 64),          # the small oracle-size case
    (2, 3, 37, 4, 64),          # ragged S_local, several planes
    (4, 2, 100, 8, 128),
    (8, 2, 53, 40, 128),        # the ragged-tail workload's heads, short sequence
    (3, 2, 29, 6, 32),          # odd rank count
    (1, 2, 33, 4, 64),          # w = 1: identity copy
    (8, 1, 7, 8, 256),          # D at the TMA box limit, H/w = 1
]

# The default (short-lived single-warp CTAs, one tile each, residency capped),
# other residency caps, then other shapes of both schedules: chunked grids
# with deeper rings or other chunk sizes, and persistent grids
# (chunk_units=0) with 1-4 producers and 2-4 stages each.
TUNINGS = [
    {},
    dict(ctas_per_sm=4),                          # residency cap: 56 KB reserved per CTA
    dict(producers=2, chunk_units=2, ctas_per_sm=7),
    dict(rows_per_tile=7, stages=2),
    dict(rows_per_tile=5, stages=12, chunk_units=7),
    dict(producers=1, chunk_units=3),
    dict(producers=3, stages=3, chunk_units=5, order=0),
    dict(rows_per_tile=16, ctas_per_sm=2, stages=3, chunk_units=0),
    dict(rows_per_tile=1, ctas_per_sm=1, stages=2, chunk_units=0),
    dict(rows_per_tile=2, stages=6, chunk_units=0),
    dict(rows_per_tile=3, stages=8, chunk_units=0, order=0),
    dict(rows_per_tile=5, ctas_per_sm=2, stages=12, chunk_units=0),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "w{}B{}S{}H{}D{}".format(*s))
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("path", [PATH_TMA, PATH_VEC], ids=["tma", "vec"])
def test_parity_small(shape, mode, path):
    w, B, S, H, D = shape
    xs = normal_slabs(slab_shape(mode, w, B, S, H, D), w, "bf16", seed0=100 + mode)
    a2a = UlyssesA2A(0, 2)
    try:
        for tuning in TUNINGS:
            for chunked in (False, True):
                run_case(xs, mode, chunked=chunked, path=path, tuning=tuning, a2a=a2a)
    finally:
        a2a.close()


@pytest.mark.parametrize("order", [0, 1])
@pytest.mark.parametrize("path", [PATH_TMA, PATH_VEC], ids=["tma", "vec"])
def test_parity_unit_orders(order, path):
    # both numberings of the work units (destination rank outermost / innermost)
    with UlyssesA2A(0, 2) as a2a:
        for (w, B, S, H, D) in [(4, 2, 37, 8, 64), (8, 2, 53, 40, 128), (3, 3, 11, 6, 32)]:
            for mode in (0, 1):
                xs = normal_slabs(slab_shape(mode, w, B, S, H, D), w, "bf16", seed0=300 + mode)
                for tuning in ({}, dict(rows_per_tile=7, stages=2, chunk_units=0),
                               dict(rows_per_tile=3, stages=8)):
                    for chunked in (False, True):
                        run_case(xs, mode, chunked=chunked, path=path,
                                 tuning=dict(tuning, order=order), a2a=a2a)


@pytest.mark.parametrize("chunk_units", [1, 5, 16])
def test_parity_chunked_grid_schedule(chunk_units):
    # TMA grid of ceil(units / n) CTAs, each taking n consecutive units
    for order in (0, 1):
        with UlyssesA2A(0, 2) as a2a:
            for (w, B, S, H, D) in [(4, 2, 37, 8, 64), (8, 1, 53, 40, 128)]:
                for mode in (0, 1):
                    xs = normal_slabs(slab_shape(mode, w, B, S, H, D), w, "bf16", seed0=400)
                    for tuning in ({}, dict(rows_per_tile=7, stages=2), dict(rows_per_tile=3, stages=8),
                                   dict(producers=2, stages=2)):
                        run_case(xs, mode, chunked=(tuning.get("stages") == 2), path=PATH_TMA,
                                 tuning=dict(tuning, chunk_units=chunk_units, order=order),
                                 a2a=a2a)


@pytest.mark.parametrize("E", [1, 2, 4, 8])
@pytest.mark.parametrize("path", [PATH_TMA, PATH_VEC], ids=["tma", "vec"])
def test_parity_unique_ids_every_element_size(E, path):
    # every element distinct: a misplaced element can never match by chance.
    # D*E = 32 bytes keeps every element size expressible by the TMA path.
    if E == 1:
        w, B, S, H, D = 2, 1, 2, 2, 32        # 256 ids fill a byte exactly
    else:
        w, B, S, H, D = 4, 2, 19, 8, 32 // E
    xs = unique_slabs((B, S, H, D), w, E)
    for mode in (0, 1):
        xin = xs if mode == 0 else oracle.ulysses_a2a(xs, 0)
        run_case(xin, mode, path=path, tuning=dict(rows_per_tile=5, stages=2))
        run_case(xin, mode, path=path, tuning=dict(rows_per_tile=1, stages=2), chunked=True)


def test_parity_fp32_uniform():
    w, B, S, H, D = 4, 2, 45, 8, 128
    for mode in (0, 1):
        xs = uniform_slabs(slab_shape(mode, w, B, S, H, D), w, "fp32", seed0=7)
        run_case(xs, mode)
        run_case(xs, mode, path=PATH_VEC)


def test_parity_rank_tagged_bf16_width():
    w, B, S, H, D = 8, 2, 33, 16, 64
    xs = rank_tagged_slabs((B, S, H, D), w)
    y = run_case(xs, 0)
    run_case(y, 1)


def test_round_trip_on_device():
    w, B, S, H, D = 4, 2, 77, 8, 64
    xs = normal_slabs((B, S, H, D), w, "bf16", seed0=5)
    with UlyssesA2A(0, 2) as a2a:
        xd = [t.cuda() for t in xs]
        y = a2a.run(xd, 0)
        z = a2a.run(y, 1)
        a2a.status()
        for k in range(w):
            assert torch.equal(bits(z[k].cpu()), bits(xs[k]))


def test_nan_payloads_and_signed_zero_survive():
    w, B, S, H, D = 2, 1, 8, 2, 8
    xs = normal_slabs((B, S, H, D), w, "fp32", seed0=9)
    b0 = xs[0].view(torch.int32)
    b0.view(-1)[0] = 0x7FC01234
    b0.view(-1)[3] = 0x7F800001
    xs[1].view(torch.int32).view(-1)[5] = -(2 ** 31)
    for path in (PATH_TMA, PATH_VEC):
        run_case(xs, 0, path=path)


# ---- alignment: misaligned slabs take the narrower vector path --------------

@pytest.mark.parametrize("offset", [8, 4, 2, 1])
def test_one_sided_offsets_take_the_shifted_vector_kernel(offset):
    # slabs off the 16-byte boundary on one side only (runs and rows of whole
    # 16-byte multiples): AUTO and the vector path forced join 16-byte vectors
    # across the two offsets (peeled = 2); the staged path, forced, re-aligns
    # in shared memory in pieces of the alignment the bases allow
    w, B, S, H, D = 2, 2, 21, 4, 64
    E = 2 if offset % 2 == 0 else 1
    if E == 2:
        xs = normal_slabs((B, S, H, D), w, "bf16", seed0=3)
    else:
        xs = random_byte_slabs((B, S, H, D * 2), w, seed0=3)
    with UlyssesA2A(0, E) as a2a:
        xd = [t.cuda() for t in xs]
        g = Guarded(oracle.output_shape(tuple(xs[0].shape), 0, w), xs[0].dtype, w, offset=offset)
        for path in (PATH_AUTO, PATH_VEC):
            a2a.set_path(path)
            plan = a2a.plan(xd, 0, out=g.slabs)
            assert plan["path"] == PATH_VEC and plan["vec_bytes"] == 16 and plan["peeled"] == 2
        a2a.set_path(PATH_STAGED)
        plan = a2a.plan(xd, 0, out=g.slabs)
        assert plan["path"] == PATH_STAGED and plan["vec_bytes"] == min(offset, 16)
    for path in (PATH_AUTO, PATH_VEC, PATH_STAGED):
        for chunked in (False, True):
            run_case(xs, 0, out_offset=offset, path=path, chunked=chunked)
            run_case(xs, 0, in_offset=offset, path=path, chunked=chunked)
            ys = oracle.ulysses_a2a(xs, 0)
            run_case(ys, 1, out_offset=offset, path=path, chunked=chunked)
            run_case(ys, 1, in_offset=offset, path=path, chunked=chunked)


def test_shapes_tma_cannot_express_use_vec():
    # D*E = 6 bytes: rows of 12 bytes; AUTO re-aligns them (staged path, 4-byte
    # pieces), and the VEC path with 4-byte vectors gives the same bytes
    w, B, S, H, D = 2, 2, 17, 4, 3
    for mode in (0, 1):
        xs = normal_slabs(slab_shape(mode, w, B, S, H, D), w, "bf16", seed0=1)
        for path in (PATH_AUTO, PATH_VEC):
            run_case(xs, mode, path=path)
            run_case(xs, mode, chunked=True, path=path)
    # w = 16 exceeds the TMA descriptor table
    w, B, S, H, D = 16, 1, 9, 16, 64
    xs = normal_slabs((B, S, H, D), w, "bf16", seed0=2)
    run_case(xs, 0)
    with pytest.raises(A2AError):
        run_case(xs, 0, path=PATH_TMA)


# ---- the benchmark's configurations at full size (default launch config) ----

FULL = {
    "w2_S64_H4_D64": (2, 1, 64, 4, 64),
    "w4_S8192_H24_D128": (4, 1, 8192, 24, 128),
    "w8_B2_S4725_H40_D128": (8, 2, 4725, 40, 128),
    "w4_B4_S16384_H32_D64": (4, 4, 16384, 32, 64),
}


@pytest.mark.parametrize("name", sorted(FULL))
def test_full_size_configs(name):
    w, B, S, H, D = FULL[name]
    xs = normal_slabs((B, S, H, D), w, "bf16")
    y = run_case(xs, 0)
    run_case(y, 1)
    if B > 1:
        run_case(xs, 0, chunked=True)
        run_case(y, 1, chunked=True)
    if name.startswith("w8_B2_S4725"):
        # the ragged tile: 4725 = 147 * 32 + 21
        run_case(xs, 0, tuning=dict(rows_per_tile=32))
        run_case(y, 1, tuning=dict(rows_per_tile=32), path=PATH_VEC)
        run_case(xs, 0, tuning=dict(rows_per_tile=32, chunk_units=0))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("w", [2, 4, 8])
def test_sweep_points(dtype, w):
    # bandwidth-sweep geometry: D = 128, H = 8w, B = 1, S_local set by the payload
    E = 2 if dtype == "bf16" else 4
    H, D = 8 * w, 128
    for payload in (256 << 10, 8 << 20, 64 << 20):
        S = payload // (w * H * D * E)
        if S < 1:
            continue
        for mode in (0, 1):
            xs = uniform_slabs(slab_shape(mode, w, 1, S, H, D), w, dtype, seed0=payload % 1000)
            run_case(xs, mode)


# ---- the host-buffer entry point -------------------------------------------

def test_run_host_matches_oracle():
    w, B, S, H, D = 4, 2, 300, 8, 128
    with UlyssesA2A(0, 2) as a2a:
        for mode in (0, 1):
            xs = normal_slabs(slab_shape(mode, w, B, S, H, D), w, "bf16", seed0=21)
            pinned = [t.pin_memory() for t in xs]
            for src in (xs, pinned):
                out = a2a.run_host(src, mode)
                want = oracle.ulysses_a2a(xs, mode)
                for k in range(w):
                    assert torch.equal(bits(out[k]), bits(want[k]))
        # the staging buffers grow on demand
        xs = normal_slabs((B, 2 * S, H, D), w, "bf16", seed0=22)
        out = a2a.run_host(xs, 0, chunked=True)
        want = oracle.ulysses_a2a(xs, 0)
        for k in range(w):
            assert torch.equal(bits(out[k]), bits(want[k]))


@pytest.mark.parametrize("path", [PATH_TMA, PATH_VEC], ids=["tma", "vec"])
def test_run_host_pipelined_chunks(path):
    # >= 8 MB of payload: the host path overlaps H2D, kernel and D2H over 8
    # sequence chunks; S_local = 1000 leaves a ragged last tile and chunk
    w, B, S, H, D = 4, 2, 1000, 8, 128
    with UlyssesA2A(0, 2) as a2a:
        a2a.set_path(path)
        for mode in (0, 1):
            xs = [t.pin_memory() for t in
                  normal_slabs(slab_shape(mode, w, B, S, H, D), w, "bf16", seed0=23 + mode)]
            want = oracle.ulysses_a2a(xs, mode)
            for chunked in (False, True):
                for knobs in ({}, dict(rows_per_tile=7), dict(chunk_units=0, rows_per_tile=13)):
                    a2a.set_tuning(**knobs)
                    n0 = a2a.launch_count
                    out = a2a.run_host(xs, mode, chunked=chunked)
                    assert a2a.launch_count - n0 > (B if chunked else 1)   # several chunks
                    for k in range(w):
                        assert torch.equal(bits(out[k]), bits(want[k])), (mode, chunked, knobs)
        a2a.status()


# ---- argument errors on a live device: nothing is launched ------------------

def test_errors_launch_nothing():
    w, B, S, H, D = 2, 1, 8, 4, 64
    with UlyssesA2A(0, 2) as a2a:
        xs = [t.cuda() for t in normal_slabs((B, S, H, D), w, "bf16")]
        outs = [torch.empty(B, S * w, H // w, D, dtype=torch.bfloat16, device="cuda")
                for _ in range(w)]
        n0 = a2a.launch_count
        # a host pointer where device memory is required
        host = [t.cpu() for t in outs]
        with pytest.raises(A2AError) as e:
            _raise(a2a, _lib.ulysses_a2a_run(a2a._ctx, [t.data_ptr() for t in xs],
                                             [t.data_ptr() for t in host], B, S, H, D, w, 0, 0, 0))
        assert e.value.code == _lib.ERR_DEVICE
        # output overlapping an input
        rc = _lib.ulysses_a2a_run(a2a._ctx, [t.data_ptr() for t in xs],
                                  [xs[0].data_ptr(), outs[1].data_ptr()], B, S, H, D, w, 0, 0, 0)
        assert rc == _lib.ERR_OVERLAP and "overlaps" in a2a.last_error()
        # H not divisible by w
        rc = _lib.ulysses_a2a_run(a2a._ctx, [t.data_ptr() for t in xs],
                                  [t.data_ptr() for t in outs], B, S, 3, D, w, 0, 0, 0)
        assert rc == _lib.ERR_INVALID
        assert a2a.launch_count == n0
        # the context still works after the rejected calls
        a2a.run(xs, 0, out=outs)
        a2a.status()
        assert a2a.launch_count == n0 + 1


def _raise(a2a, rc):
    if rc != _lib.OK:
        raise A2AError(rc, a2a.last_error())


def test_slab_past_end_of_allocation_is_rejected():
    from cuda.bindings import runtime as rt

    w, B, S, H, D = 2, 1, 64, 4, 64
    nbytes = B * S * H * D * 2
    size = 4 << 20
    err, base = rt.cudaMalloc(size)            # a dedicated allocation of known extent
    assert err == rt.cudaError_t.cudaSuccess
    try:
        with UlyssesA2A(0, 2) as a2a:
            xs = [t.cuda() for t in normal_slabs((B, S, H, D), w, "bf16")]
            out0 = torch.empty(B, S * w, H // w, D, dtype=torch.bfloat16, device="cuda")
            n0 = a2a.launch_count
            # second output starts half a slab before the allocation's end
            rc = _lib.ulysses_a2a_run(a2a._ctx, [t.data_ptr() for t in xs],
                                      [out0.data_ptr(), int(base) + size - nbytes // 2],
                                      B, S, H, D, w, 0, 0, 0)
            assert rc == _lib.ERR_DEVICE and "past the end" in a2a.last_error()
            # the same slab placed wholly inside the allocation is accepted
            rc = _lib.ulysses_a2a_run(a2a._ctx, [t.data_ptr() for t in xs],
                                      [out0.data_ptr(), int(base) + size - nbytes],
                                      B, S, H, D, w, 0, 0, 0)
            assert rc == _lib.OK
            a2a.status()
            assert a2a.launch_count == n0 + 1
    finally:
        torch.cuda.synchronize()
        rt.cudaFree(base)


def test_status_is_clean_and_destroy_is_idempotent_on_null():
    a2a = UlyssesA2A(0, 2)
    xs = [t.cuda() for t in normal_slabs((1, 16, 4, 64), 2, "bf16")]
    a2a.run(xs, 0)
    a2a.status()
    a2a.close()
    a2a.close()
    assert _lib.lib.ulysses_a2a_destroy(None) == _lib.OK


# ---- the autograd pairing: backward of mode m is mode 1-m -------------------

@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_autograd_backward_is_the_inverse_mode(mode, dtype):
    from sequence_all_re_b200.autograd import all_to_all_4d

    w, B, S, H, D = 4, 2, 29, 8, 64
    E = 2 if dtype == "bf16" else 4
    xs = normal_slabs(slab_shape(mode, w, B, S, H, D), w, dtype, seed0=500)
    # upstream gradient: one seeded weight tensor per output slab
    cs = normal_slabs(slab_shape(1 - mode, w, B, S, H, D), w, dtype, seed0=600)
    with UlyssesA2A(0, E) as a2a:
        xd = [t.cuda().requires_grad_(True) for t in xs]
        ys = all_to_all_4d(a2a, xd, mode, chunked=(mode == 1))
        loss = sum((y.float() * c.cuda().float()).sum() for y, c in zip(ys, cs))
        loss.backward()
        a2a.status()
        want_y = oracle.ulysses_a2a(xs, mode)
        want_g = oracle.ulysses_a2a(cs, 1 - mode)     # P^-1 applied to the weights
        for k in range(w):
            assert torch.equal(bits(ys[k].detach().cpu()), bits(want_y[k]))
            assert torch.equal(bits(xd[k].grad.cpu()), bits(want_g[k]))


def test_autograd_unused_outputs_get_zero_gradient():
    from sequence_all_re_b200.autograd import all_to_all_4d

    w, B, S, H, D = 2, 1, 16, 4, 64
    xs = normal_slabs((B, S, H, D), w, "fp32", seed0=7)
    with UlyssesA2A(0, 4) as a2a:
        xd = [t.cuda().requires_grad_(True) for t in xs]
        ys = all_to_all_4d(a2a, xd, 0)
        ys[1].sum().backward()          # only rank 1's output is used
        ones_then_zero = [torch.zeros_like(ys[0]).cpu(), torch.ones_like(ys[1]).cpu()]
        want = oracle.ulysses_a2a(ones_then_zero, 1)
        for k in range(w):
            assert torch.equal(xd[k].grad.cpu(), want[k])


# ---- CUDA graph capture of the C-ABI call -----------------------------------

def test_run_captures_into_a_cuda_graph():
    w, B, S, H, D = 4, 2, 37, 8, 64
    xs = normal_slabs((B, S, H, D), w, "bf16", seed0=31)
    want = oracle.ulysses_a2a(xs, 0)
    back = oracle.ulysses_a2a(want, 1)
    with UlyssesA2A(0, 2) as a2a:
        xd = [t.cuda() for t in xs]
        yd = [torch.empty(B, S * w, H // w, D, dtype=torch.bfloat16, device="cuda") for _ in range(w)]
        zd = [torch.empty_like(t) for t in xd]
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):                 # warm-up outside capture
            a2a.run(xd, 0, out=yd, stream=s)
            a2a.run(yd, 1, out=zd, stream=s, chunked=True)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            a2a.run(xd, 0, out=yd)
            a2a.run(yd, 1, out=zd, chunked=True)
        for t in yd + zd:
            t.view(torch.int16).fill_(-1)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        a2a.status()
        for k in range(w):
            assert torch.equal(bits(yd[k].cpu()), bits(want[k]))
            assert torch.equal(bits(zd[k].cpu()), bits(back[k]))
        del g


# ---- row-pitched [B, S, H, D] side: packed QKV projection layouts -----------

@pytest.mark.parametrize("path", [PATH_TMA, PATH_VEC], ids=["tma", "vec"])
def test_packed_qkv_mode0_reads_in_place(path):
    w, B, S, H, D = 4, 2, 37, 8, 64
    packed_cpu = normal_slabs((B, S, 3, H, D), w, "bf16", seed0=700)
    flat = [t.reshape(-1) for t in packed_cpu]
    with UlyssesA2A(0, 2) as a2a:
        a2a.set_path(path)
        packed = [t.cuda() for t in packed_cpu]
        for c in range(3):                                # q, k, v
            want = oracle.ulysses_a2a_pitched(flat, 0, w, B, S, H, D, 3 * H * D, offset=c * H * D)
            views = [t[:, :, c] for t in packed]          # strides (S*3HD, 3HD, D, 1)
            assert views[0].stride() == (S * 3 * H * D, 3 * H * D, D, 1)
            for chunked in (False, True):
                for knobs in ({}, dict(rows_per_tile=5, chunk_units=0)):
                    a2a.set_tuning(**knobs)
                    assert a2a.plan(views, 0, knobs=knobs)["row_pitch"] == 3 * H * D
                    out = a2a.run(views, 0, chunked=chunked)
                    for r in range(w):
                        assert torch.equal(bits(out[r].cpu()).reshape(-1), bits(want[r])), (c, r)
        a2a.status()


@pytest.mark.parametrize("path", [PATH_TMA, PATH_VEC], ids=["tma", "vec"])
def test_mode1_writes_into_packed_slots(path):
    w, B, S, H, D = 4, 2, 29, 8, 64
    with UlyssesA2A(0, 2) as a2a:
        a2a.set_path(path)
        ys = [normal_slabs((B, S * w, H // w, D), w, "bf16", seed0=710 + c) for c in range(3)]
        packed = [torch.empty((B, S, 3, H, D), dtype=torch.bfloat16, device="cuda")
                  for _ in range(w)]
        for t in packed:
            t.view(torch.int16).fill_(-1)
        # write only slot 1 (k) first: slots 0 and 2 keep their poison
        a2a.run([y.cuda() for y in ys[1]], 1, out=[t[:, :, 1] for t in packed])
        torch.cuda.synchronize()
        want1 = oracle.ulysses_a2a(ys[1], 1)
        for j in range(w):
            got = packed[j].cpu()
            assert torch.equal(bits(got[:, :, 1].contiguous()), bits(want1[j]))
            assert bool((got[:, :, 0].view(torch.int16) == -1).all())
            assert bool((got[:, :, 2].view(torch.int16) == -1).all())
        for c in (0, 2):
            a2a.run([y.cuda() for y in ys[c]], 1, out=[t[:, :, c] for t in packed], chunked=True)
        a2a.status()
        for c in range(3):
            want = oracle.ulysses_a2a(ys[c], 1)
            for j in range(w):
                assert torch.equal(bits(packed[j][:, :, c].cpu().contiguous()), bits(want[j]))


@pytest.mark.parametrize("path", [PATH_AUTO, PATH_VEC, PATH_STAGED], ids=["auto", "vec", "staged"])
def test_odd_row_pitch_uses_narrower_pieces(path):
    # rows of H*D + 4 bf16 elements: 8-byte aligned only, so 8-byte vectors
    # (VEC, also AUTO's choice) or 8-byte pieces (staged, forced); the 4
    # trailing elements of every row stay untouched
    w, B, S, H, D = 2, 2, 19, 4, 32
    pitch = H * D + 4
    bufs_cpu = normal_slabs((B * S * pitch,), w, "bf16", seed0=720)
    want = oracle.ulysses_a2a_pitched(bufs_cpu, 0, w, B, S, H, D, pitch)
    with UlyssesA2A(0, 2) as a2a:
        a2a.set_path(path)
        bufs = [t.cuda() for t in bufs_cpu]
        views = [t.as_strided((B, S, H, D), (S * pitch, pitch, D, 1)) for t in bufs]
        p = a2a.plan(views, 0)
        assert p["path"] == (PATH_STAGED if path == PATH_STAGED else PATH_VEC)
        assert p["vec_bytes"] == 8 and p["row_pitch"] == pitch
        out = a2a.run(views, 0)
        for r in range(w):
            assert torch.equal(bits(out[r].cpu()).reshape(-1), bits(want[r]))
        # and back: mode 1 into the pitched buffers leaves the gaps alone
        dst = [torch.full_like(t, float("nan")) for t in bufs]
        a2a.run(out, 1, out=[t.as_strided((B, S, H, D), (S * pitch, pitch, D, 1)) for t in dst])
        a2a.status()
        for j in range(w):
            got = dst[j].cpu().view(B * S, pitch)
            src = bufs_cpu[j].view(B * S, pitch)
            assert torch.equal(bits(got[:, :H * D].contiguous()), bits(src[:, :H * D].contiguous()))
            assert bool(torch.isnan(got[:, H * D:].float()).all())


# ---- failure detection: a bounded wait that expires ---------------------------

def test_bounded_wait_expiry_is_reported_and_context_survives():
    # the self-test kernel waits on an mbarrier nothing arrives on (50 ms limit)
    from sequence_all_re_b200 import _lib as L

    with UlyssesA2A(0, 2) as a2a:
        a2a.status()                                       # clean to start with
        stream = torch.cuda.current_stream()
        rc = L.lib.ulysses_a2a_selftest_wait_timeout(a2a._ctx, 50000, stream.cuda_stream)
        assert rc == L.OK
        with pytest.raises(A2AError) as e:
            a2a.status()
        assert e.value.code == L.ERR_TIMEOUT and "gave up" in a2a.last_error()
        a2a.status()                                       # reading it cleared it
        # the context and the device still work
        run_case(normal_slabs((1, 16, 4, 64), 2, "bf16", seed0=3), 0, a2a=a2a)
        rc = L.lib.ulysses_a2a_selftest_wait_timeout(a2a._ctx, 0, stream.cuda_stream)
        assert rc == L.ERR_INVALID


# ---- chunked = 2: per plane through the context's staging window -------------

@pytest.mark.parametrize("path", [PATH_TMA, PATH_VEC], ids=["tma", "vec"])
def test_windowed_chunked_variant(path):
    with UlyssesA2A(0, 2) as a2a:
        a2a.set_path(path)
        # small first, then larger planes: the window grows on demand
        for (w, B, S, H, D) in [(2, 2, 9, 4, 64), (4, 3, 37, 8, 64), (8, 2, 53, 40, 128)]:
            for mode in (0, 1):
                xs = normal_slabs(slab_shape(mode, w, B, S, H, D), w, "bf16", seed0=800 + mode)
                run_case(xs, mode, chunked=2, path=path, a2a=a2a)
        # packed QKV input read through the window
        w, B, S, H, D = 4, 2, 21, 8, 64
        packed_cpu = normal_slabs((B, S, 3, H, D), w, "bf16", seed0=810)
        want = oracle.ulysses_a2a_pitched([t.reshape(-1) for t in packed_cpu], 0, w, B, S, H, D,
                                          3 * H * D, offset=H * D)
        packed = [t.cuda() for t in packed_cpu]
        out = a2a.run([t[:, :, 1] for t in packed], 0, chunked=2)
        for r in range(w):
            assert torch.equal(bits(out[r].cpu()).reshape(-1), bits(want[r]))
        a2a.status()


def test_windowed_variant_is_refused_where_no_window_exists():
    w, B, S, H, D = 2, 2, 8, 4, 64
    xs = normal_slabs((B, S, H, D), w, "bf16")
    with UlyssesA2A(0, 2) as a2a:
        with pytest.raises(A2AError) as e:
            a2a.run_host(xs, 0, chunked=2)
        assert e.value.code == _lib.ERR_UNSUPPORTED
    xd = [t.cuda() for t in xs]
    yd = [torch.empty(B, S * w, H // w, D, dtype=torch.bfloat16, device="cuda") for _ in range(w)]
    rc, msg = _lib.ulysses_a2a_run_noalloc([t.data_ptr() for t in xd], [t.data_ptr() for t in yd],
                                           B, S, H, D, w, 0, 2, 2,
                                           torch.cuda.current_stream().cuda_stream)
    assert rc == _lib.ERR_UNSUPPORTED and "window" in msg


# ---- randomized coverage ------------------------------------------------------

def test_randomized_shapes_layouts_and_knobs():
    """150 seeded random cases: w in 1..16, ragged S_local, odd D, element sizes
    1/2/4/8, both modes, chunked 0/1/2, random row pitches on the [B,S,H,D] side
    (gap bytes must survive), random tuning and both paths; bit-exact against
    the oracle every time."""
    import random

    rng = random.Random(20241202)
    INT = {1: torch.uint8, 2: torch.int16, 4: torch.int32, 8: torch.int64}
    ctxs = {E: UlyssesA2A(0, E) for E in (1, 2, 4, 8)}
    try:
        for case in range(150):
            w = rng.choice([1, 2, 3, 4, 5, 8, 12, 16])
            B, S = rng.randint(1, 3), rng.randint(1, 70)
            H = w * rng.randint(1, 4)
            D = rng.choice([1, 3, 8, 16, 24, 64, 128, 200, 256])
            E = rng.choice([1, 2, 4, 8])
            mode, chunked = rng.randint(0, 1), rng.choice([0, 0, 1, 2])
            pitch = H * D + rng.choice([0, 0, 0, rng.randint(1, 40), 8 * rng.randint(1, 6)])
            knobs = {}
            if rng.random() < 0.6:
                knobs = dict(rows_per_tile=rng.randint(0, 9), stages=rng.choice([0, 2, 3, 4, 8, 12]),
                             chunk_units=rng.choice([-1, 0, 1, 3, 7]), order=rng.choice([-1, 0, 1]),
                             producers=rng.choice([0, 1, 2, 3, 4, 8]))
            path = rng.choice([PATH_AUTO, PATH_AUTO, PATH_VEC, PATH_STAGED])
            if path == PATH_STAGED and H * D * E > 90 * 1024:
                path = PATH_AUTO            # one row would not fit the staged path's shared memory
            a2a = ctxs[E]
            a2a.set_path(path)
            a2a.set_tuning(**knobs)
            dt = INT[E]
            n_pitched = (B * S - 1) * pitch + H * D
            n_dense = B * S * H * D
            seed = 9000 + case
            if mode == 0:
                bufs = [t.view(dt) for t in random_byte_slabs((n_pitched * E,), w, seed0=seed)]
                want = oracle.ulysses_a2a_pitched(bufs, 0, w, B, S, H, D, pitch)
                dev = [t.cuda() for t in bufs]
                xs = [t.as_strided((B, S, H, D), (S * pitch, pitch, D, 1)) for t in dev]
                out = [torch.empty(B, S * w, H // w, D, dtype=dt, device="cuda") for _ in range(w)]
                for o in out:
                    o.view(torch.uint8).fill_(0xFF)
                a2a.run(xs, 0, chunked=chunked, out=out)
                got = [o.cpu().reshape(-1) for o in out]
            else:
                ins = [t.view(dt) for t in random_byte_slabs((n_dense * E,), w, seed0=seed)]
                poison = [torch.full((n_pitched * E,), 0xA5, dtype=torch.uint8).view(dt)
                          for _ in range(w)]
                want = oracle.ulysses_a2a_pitched(ins, 1, w, B, S, H, D, pitch,
                                                  out_bufs=[p.clone() for p in poison])
                xs = [t.cuda().view(B, S * w, H // w, D) for t in ins]
                dst = [p.cuda() for p in poison]
                out = [t.as_strided((B, S, H, D), (S * pitch, pitch, D, 1)) for t in dst]
                a2a.run(xs, 1, chunked=chunked, out=out)
                got = [t.cpu() for t in dst]
            a2a.status()
            for k in range(w):
                assert torch.equal(got[k], want[k].reshape(-1)), (
                    f"case {case}: w={w} B={B} S={S} H={H} D={D} E={E} mode={mode} "
                    f"chunked={chunked} pitch={pitch} path={path} knobs={knobs} rank={k}")
    finally:
        for c in ctxs.values():
            c.close()


def test_two_contexts_on_two_streams_concurrently():
    # independent contexts and streams: results must not interfere
    w, B, S, H, D = 4, 2, 300, 8, 128
    xa = normal_slabs((B, S, H, D), w, "bf16", seed0=901)
    xb = normal_slabs((B, S * w, H // w, D), w, "bf16", seed0=902)
    wa, wb = oracle.ulysses_a2a(xa, 0), oracle.ulysses_a2a(xb, 1)
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    with UlyssesA2A(0, 2) as c1, UlyssesA2A(0, 2) as c2:
        c2.set_path(PATH_VEC)
        da, db = [t.cuda() for t in xa], [t.cuda() for t in xb]
        ya = [torch.empty(B, S * w, H // w, D, dtype=torch.bfloat16, device="cuda") for _ in range(w)]
        yb = [torch.empty(B, S, H, D, dtype=torch.bfloat16, device="cuda") for _ in range(w)]
        torch.cuda.synchronize()
        for _ in range(20):
            c1.run(da, 0, out=ya, stream=sa)
            c2.run(db, 1, out=yb, stream=sb, chunked=True)
        c1.status(sa)
        c2.status(sb)
        for k in range(w):
            assert torch.equal(bits(ya[k].cpu()), bits(wa[k]))
            assert torch.equal(bits(yb[k].cpu()), bits(wb[k]))


def test_default_stream_is_torchs_current_stream():
    # run() without a stream queues on torch's current stream, inside a
    # `torch.cuda.stream` block too: it must see the inputs written there after
    # a long kernel on that stream (on any other stream it would read them early)
    w, B, S, H, D = 2, 1, 64, 4, 128
    cpu = normal_slabs((B, S, H, D), w, "bf16", seed0=911)
    want = oracle.ulysses_a2a(cpu, 0)
    s = torch.cuda.Stream()
    with UlyssesA2A(0, 2) as a2a:
        assert a2a._stream_handle(None) == torch.cuda.current_stream().cuda_stream
        xs = [torch.zeros(B, S, H, D, dtype=torch.bfloat16, device="cuda") for _ in range(w)]
        staged = [c.cuda() for c in cpu]
        torch.cuda.synchronize()
        with torch.cuda.stream(s):
            assert a2a._stream_handle(None) == s.cuda_stream
            torch.cuda._sleep(20_000_000)
            for x, c in zip(xs, staged):
                x.copy_(c)
            ys = a2a.run(xs, 0)
        s.synchronize()
        a2a.status(s)
        for k in range(w):
            assert torch.equal(bits(ys[k].cpu()), bits(want[k]))


def test_bound_calls_follow_the_slabs_contents():
    # bind once, call many times: each call re-lays out the slabs' current
    # contents; a chunked binding launches once per plane
    w, B, S, H, D = 4, 3, 77, 8, 64
    with UlyssesA2A(0, 2) as a2a:
        xs = [torch.empty(B, S, H, D, dtype=torch.bfloat16, device="cuda") for _ in range(w)]
        for chunked in (False, True):
            call = a2a.bind(xs, 0, chunked=chunked)
            for seed in (931, 932):
                cpu = normal_slabs((B, S, H, D), w, "bf16", seed0=seed)
                for x, c in zip(xs, cpu):
                    x.copy_(c)
                n0 = a2a.launch_count
                ys = call()
                assert a2a.launch_count - n0 == (B if chunked else 1)
                a2a.status()
                want = oracle.ulysses_a2a(cpu, 0)
                for r in range(w):
                    assert torch.equal(bits(ys[r].cpu()), bits(want[r])), (chunked, seed, r)
        # mode 1 back into row-pitched q slots of a packed buffer
        pitch = 3 * H * D
        packed = torch.full((w, B * S * pitch), float("nan"), dtype=torch.bfloat16, device="cuda")
        views = [packed[k].as_strided((B, S, H, D), (S * pitch, pitch, D, 1)) for k in range(w)]
        back = a2a.bind(ys, 1, out=views)
        assert back() is back.out
        a2a.status()
        for j in range(w):
            assert torch.equal(bits(views[j].cpu()), bits(cpu[j]))


def test_bound_call_refuses_a_reallocated_slab():
    w, B, S, H, D = 2, 1, 16, 4, 64
    with UlyssesA2A(0, 2) as a2a:
        xs = [torch.zeros(B, S, H, D, dtype=torch.bfloat16, device="cuda") for _ in range(w)]
        call = a2a.bind(xs, 0)
        call()
        n0 = a2a.launch_count
        xs[1].set_(torch.zeros(B, S, H, D, dtype=torch.bfloat16, device="cuda"))
        with pytest.raises(ValueError, match="reallocated"):
            call()
        call = a2a.bind(xs, 0)                              # an output slab, this time
        call()
        n0 = a2a.launch_count
        out = call.out[0]
        out.resize_(2 * out.numel())                        # grows: a new allocation
        with pytest.raises(ValueError, match="reallocated"):
            call()
        assert a2a.launch_count == n0                       # nothing was launched
        a2a.status()


# ---- edge sizes: empty, maximum rank count, box limits, a 2 GiB payload -------

def test_empty_relayouts_launch_nothing():
    with UlyssesA2A(0, 2) as a2a:
        for shape, mode in [((0, 8, 4, 64), 0), ((2, 0, 4, 64), 0), ((2, 8, 4, 0), 0),
                            ((2, 0, 2, 64), 1)]:
            xs = [torch.empty(shape, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
            for chunked in (0, 1, 2):
                n0 = a2a.launch_count
                ys = a2a.run(xs, mode, chunked=chunked)
                assert a2a.launch_count == n0
                assert all(y.numel() == 0 for y in ys)
                assert tuple(ys[0].shape) == oracle.output_shape(shape, mode, 2)
            hs = a2a.run_host([x.cpu() for x in xs], mode)
            assert all(h.numel() == 0 for h in hs)
        a2a.status()
    rc, msg = _lib.ulysses_a2a_run_noalloc([0, 0], [0, 0], 0, 8, 4, 64, 2, 0, 0, 2,
                                           torch.cuda.current_stream().cuda_stream)
    assert rc == _lib.OK, msg


def test_maximum_rank_count():
    w, B, S, H, D = 64, 1, 3, 64, 16            # ULYSSES_A2A_MAX_W ranks
    for mode in (0, 1):
        xs = unique_slabs(slab_shape(mode, w, B, S, H, D), w, 4)
        run_case(xs, mode)
        run_case(xs, mode, chunked=2)


def test_tma_box_and_tile_limits():
    # H/w = 128 heads x D = 256 bf16: one 64 KB row per tile, the largest TMA tile
    w, B, S, H, D = 2, 2, 5, 256, 256
    with UlyssesA2A(0, 2) as a2a:
        xs = normal_slabs((B, S, H, D), w, "bf16", seed0=950)
        a2a.set_path(PATH_TMA)      # (AUTO would take the vector kernel for so small a call)
        p = a2a.plan([t.cuda() for t in xs], 0)
        assert p["path"] == PATH_TMA and p["rows_per_tile"] == 1 and p["row_bytes"] == 64 * 1024
        for mode, x in ((0, xs), (1, oracle.ulysses_a2a(xs, 0))):
            run_case(x, mode, a2a=a2a, path=PATH_TMA)
            run_case(x, mode, a2a=a2a, path=PATH_TMA, tuning=dict(chunk_units=0))
    # rows just over the tile limit go to the VEC path
    w, B, S, H, D = 2, 1, 3, 264, 256
    xs = normal_slabs((B, S, H, D), w, "bf16", seed0=951)
    run_case(xs, 0)


def test_two_gib_payload_full_compare():
    # w = 8, H = 64, D = 128, S_local = 16384: 2 GiB of bf16 per call
    w, B, S, H, D = 8, 1, 16384, 64, 128
    xs = uniform_slabs((B, S, H, D), w, "bf16", seed0=960)
    y = run_case(xs, 0)
    del xs
    run_case(y, 1)


def _big_slabs(shape, w, offset, seed0):
    """w seeded random int16 slabs of `shape` viewed as bf16, each `offset` bytes
    into its own allocation, drawn on the device (4 GiB slabs are too large to
    draw on the host and copy)."""
    n = 2
    for v in shape:
        n *= v
    out = []
    for k in range(w):
        raw = torch.empty(n + offset, dtype=torch.uint8, device="cuda")
        t = raw[offset:].view(torch.int16).view(shape)
        g = torch.Generator(device="cuda")
        g.manual_seed(seed0 + k)
        t.random_(-32768, 32767, generator=g)
        out.append(t.view(torch.bfloat16))
    return out


@pytest.mark.parametrize("path, in_off, out_off", [
    (PATH_AUTO, 0, 0), (PATH_VEC, 0, 0), (PATH_STAGED, 0, 0),
    (PATH_AUTO, 2, 2), (PATH_AUTO, 2, 0)],
    ids=["tma", "vec", "staged", "peeled", "shifted"])
def test_slabs_over_4_gib(path, in_off, out_off):
    # w = 2, B = 2, S_local = 2^19 + 3 (ragged), H = 16, D = 128, bf16: every
    # slab is 4 GiB + 24 KB, so byte offsets inside a slab pass 2^32; the
    # kernels' address arithmetic must be 64-bit throughout. Expected rows come
    # from the oracle on one-row sub-slabs (the map sends row (b, s) of every
    # x_j to rows (b, j*S_local + s) of the outputs); the round trip is checked
    # in full on the device.
    w, B, S, H, D = 2, 2, (1 << 19) + 3, 16, 128
    Hw = H // w
    xs = _big_slabs((B, S, H, D), w, in_off, seed0=980)
    assert xs[0].numel() * 2 > (1 << 32)
    with UlyssesA2A(0, 2) as a2a:
        a2a.set_path(path)
        ys = _big_slabs((B, S * w, Hw, D), w, out_off, seed0=990)
        p = a2a.plan(xs, 0, out=ys)
        assert p["peeled"] == (0 if not in_off else (1 if in_off == out_off else 2))
        a2a.run(xs, 0, out=ys)
        a2a.status()
        g = torch.Generator().manual_seed(970)
        rows = [(int(torch.randint(0, B, (1,), generator=g)), int(torch.randint(0, S, (1,), generator=g)))
                for _ in range(24)] + [(B - 1, S - 1), (0, 0), (1, S // 2)]
        for b, s in rows:
            sub = [x[b:b + 1, s:s + 1].cpu() for x in xs]
            want = oracle.ulysses_a2a(sub, 0)          # out_r[0, j, h', d]
            for r in range(w):
                got = ys[r][b, [j * S + s for j in range(w)]].cpu().unsqueeze(0)
                assert torch.equal(bits(got), bits(want[r])), (b, s, r)
        zs = _big_slabs((B, S, H, D), w, in_off, seed0=995)
        a2a.run(ys, 1, out=zs)
        a2a.status()
        for k in range(w):
            assert torch.equal(zs[k].view(torch.int16), xs[k].view(torch.int16)), k
    del xs, ys, zs
    torch.cuda.empty_cache()


def test_environment_overrides_set_the_initial_knobs(monkeypatch):
    monkeypatch.setenv("ULYSSES_A2A_FORCE_PATH", "vec")
    monkeypatch.setenv("ULYSSES_A2A_CTAS_PER_SM", "8")
    with UlyssesA2A(0, 2) as a2a:
        monkeypatch.delenv("ULYSSES_A2A_FORCE_PATH")
        monkeypatch.delenv("ULYSSES_A2A_CTAS_PER_SM")
        path, knobs = a2a.settings()
        assert path == PATH_VEC and knobs["ctas_per_sm"] == 8
        xs = normal_slabs((1, 96, 8, 64), 4, "bf16")
        out = run_case(xs, 0, a2a=a2a, path=PATH_VEC, tuning={"ctas_per_sm": 8})
        p = a2a.plan([t.cuda() for t in xs], 0)
        assert p["path"] == PATH_VEC and p["grid"] <= 148 * 8
        # the API overrides the environment
        a2a.set_path(PATH_AUTO)
        a2a.set_tuning()
        assert a2a.settings() == (PATH_AUTO, dict(_lib.TuningT.DEFAULTS))
        p = a2a.plan([t.cuda() for t in xs], 0)      # 768 KiB: AUTO's vector kernel
        assert p["path"] == PATH_VEC and p["grid"] == p["units"]
        big = [torch.empty((1, 65536, 8, 64), dtype=torch.bfloat16, device="cuda") for _ in range(4)]
        assert a2a.plan(big, 0)["path"] == PATH_TMA   # 256 MiB: TMA
        del big
        del out


# ---- head-packed tensors in one launch ---------------------------------------

PACKED = [
    # (T, w, B, S_local, H, D)
    (3, 4, 2, 37, 8, 64),       # q, k, v; ragged S_local
    (2, 2, 1, 100, 4, 128),
    (3, 8, 1, 53, 40, 128),     # the ragged-tail workload's heads
    (3, 4, 2, 19, 4, 13),       # odd D: narrow vectors
    (1, 4, 1, 64, 8, 64),       # T = 1: the plain re-layout
]


@pytest.mark.parametrize("case", PACKED, ids=lambda c: "T{}w{}B{}S{}H{}D{}".format(*c))
@pytest.mark.parametrize("chunked", [False, True], ids=["whole", "per_plane"])
def test_packed_tensors_in_one_launch(case, chunked):
    T, w, B, S, H, D = case
    packed_cpu = normal_slabs((B, S, T, H, D), w, "bf16", seed0=900 + T)
    flat = [t.reshape(-1) for t in packed_cpu]
    with UlyssesA2A(0, 2) as a2a:
        packed = [t.cuda() for t in packed_cpu]
        n0 = a2a.launch_count
        outs = a2a.run_packed(packed, 0, chunked=chunked)
        assert a2a.launch_count - n0 == (B if chunked else 1)
        for t in range(T):
            # tensor t of the packed slabs: a row-pitched view, T*H*D between rows
            want = oracle.ulysses_a2a_pitched(flat, 0, w, B, S, H, D, T * H * D, offset=t * H * D)
            for r in range(w):
                assert torch.equal(bits(outs[t][r].cpu()).reshape(-1), bits(want[r])), (t, r)
        # mode 1 back into poisoned packed buffers, one launch (per plane when chunked)
        back = [torch.full((B, S, T, H, D), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
                for _ in range(w)]
        n1 = a2a.launch_count
        a2a.run_packed(outs, 1, chunked=chunked, out=back)
        a2a.status()
        assert a2a.launch_count - n1 == (B if chunked else 1)
        for j in range(w):
            assert torch.equal(bits(back[j].cpu()), bits(packed_cpu[j])), j


def test_packed_autograd_backward_is_packed_mode1():
    from sequence_all_re_b200.autograd import all_to_all_4d_packed

    T, w, B, S, H, D = 3, 4, 1, 45, 8, 64
    packed_cpu = normal_slabs((B, S, T, H, D), w, "bf16", seed0=950)
    gys = [uniform_slabs((B, S * w, H // w, D), w, "bf16", seed0=960 + t) for t in range(T)]
    with UlyssesA2A(0, 2) as a2a:
        xs = [t.cuda().requires_grad_() for t in packed_cpu]
        outs = all_to_all_4d_packed(a2a, xs)
        torch.autograd.backward([o for per_t in outs for o in per_t],
                                [g.cuda() for per_t in gys for g in per_t])
        # the gradient of packed slab j: tensor t's mode-1 result in slot t
        for t in range(T):
            want = oracle.ulysses_a2a(gys[t], 1)
            for j in range(w):
                assert torch.equal(bits(xs[j].grad[:, :, t].cpu().contiguous()), bits(want[j]))


def test_randomized_packed_launches():
    """Seeded random head-packed launches: T, w, shapes, element size, chunking."""
    import random

    rng = random.Random(4242)
    with UlyssesA2A(0, 2) as a2, UlyssesA2A(0, 4) as a4, UlyssesA2A(0, 1) as a1:
        ctx_of = {1: a1, 2: a2, 4: a4}
        for case in range(40):
            E = rng.choice([1, 2, 4])
            w = rng.choice([1, 2, 3, 4, 8])
            T = rng.randint(1, min(4, 64 // w))
            Hw = rng.choice([1, 2, 3, 5])
            H, B = Hw * w, rng.randint(1, 3)
            S = rng.randint(1, 70)
            D = rng.choice([1, 7, 16, 33, 64])
            chunked = rng.random() < 0.5
            dtype = {1: torch.uint8, 2: torch.int16, 4: torch.int32}[E]
            packed_cpu = random_byte_slabs((B, S, T, H, D * E), w, seed0=5000 + case)
            packed_cpu = [t.view(dtype).reshape(B, S, T, H, D) for t in packed_cpu]
            a2a = ctx_of[E]
            packed = [t.cuda() for t in packed_cpu]
            outs = a2a.run_packed(packed, 0, chunked=chunked)
            flat = [t.reshape(-1) for t in packed_cpu]
            for t in range(T):
                want = oracle.ulysses_a2a_pitched(flat, 0, w, B, S, H, D, T * H * D,
                                                  offset=t * H * D)
                for r in range(w):
                    assert torch.equal(outs[t][r].cpu().reshape(-1), want[r]), (case, t, r)
            back = a2a.run_packed(outs, 1, chunked=not chunked)
            for j in range(w):
                assert torch.equal(back[j].cpu(), packed_cpu[j]), (case, j)
        for a in (a1, a2, a4):
            a.status()
