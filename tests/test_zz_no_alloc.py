"""The allocation-free entry point, ulysses_a2a_run_noalloc (needs a B200).

Some callers cannot allocate device memory (their process's device memory is
owned by another allocator under a fixed budget, or they run where cudaMalloc
is not allowed). For them the library offers one entry point that allocates
nothing: it keeps the copy kernel's status records in a static device array.
These tests call it through the C ABI, on two calls in a row, and check every
output byte against the CPU oracle's element map and against the regular entry
point's output (bit for bit, the tolerance every test here uses). They also
check that it rejects a TMA-path chunked call needing more status records than
the array holds, while a staged- or vector-path chunked call over as many
planes needs no record and runs. This file is named so pytest collects it last; it also passes
when run alone in a fresh process (its first call does the per-device set-up).
"""

import pytest
import torch

import oracle
from sequence_all_re_b200 import UlyssesA2A, _lib
from synth import normal_slabs, slab_shape, uniform_slabs

pytestmark = pytest.mark.gpu

INT_OF = {2: torch.int16, 4: torch.int32}

TMA, VEC, STAGED = _lib.PATH_TMA, _lib.PATH_VEC, _lib.PATH_STAGED
CASES = [
    # (w, B, S_local, H, D, dtype, chunked, base offset in bytes, the path AUTO takes)
    (4, 1, 8192, 24, 128, "bf16", 0, 0, TMA),
    (8, 2, 4725, 40, 128, "bf16", 1, 0, TMA),     # chunked, ragged tail
    (4, 1, 16384, 8, 128, "fp32", 0, 0, TMA),     # fp32 (256 MiB)
    (2, 3, 37, 4, 64, "bf16", 1, 0, VEC),         # small calls: the vector kernel, chunked
    (4, 2, 45, 8, 128, "fp32", 0, 0, VEC),        # fp32
    (16, 2, 19, 16, 64, "bf16", 0, 0, VEC),       # w = 16: the vector path
    (16, 3, 19, 16, 64, "bf16", 1, 0, VEC),       # the vector path, chunked
    (2, 2, 17, 4, 3, "bf16", 0, 0, STAGED),       # 12-byte runs: re-aligned in shared memory
    (2, 3, 17, 4, 3, "bf16", 1, 0, STAGED),       # chunked
    (4, 2, 33, 4, 4, "bf16", 0, 0, STAGED),       # 8-byte runs: the fixed-phase form
    (4, 2, 33, 8, 64, "bf16", 0, 2, VEC),         # every slab 2 bytes off 16: peeled vectors
    (4, 2, 33, 8, 64, "bf16", 1, 8, VEC),         # chunked, 8 bytes off: peeled vectors
    (4, 2, 33, 8, 64, "bf16", 1, (6, 0), VEC),    # inputs 6 bytes off, outputs aligned: joined
]


def _offsets(off):
    """(input offset, output offset) of a case: one number for both, or a pair."""
    return off if isinstance(off, tuple) else (off, off)


def _device_slabs(cpu_slabs, offset):
    """Copies of the CPU slabs on the GPU, each starting `offset` bytes into its
    own allocation (a base address off the 16-byte boundary when offset > 0)."""
    out = []
    for t in cpu_slabs:
        n = t.numel() * t.element_size()
        raw = torch.empty(n + offset, dtype=torch.uint8, device="cuda")
        d = raw[offset:].view(t.dtype).view(t.shape)
        d.copy_(t)
        out.append(d)
    return out


def _poisoned(shape, dtype, w, offset):
    outs = _device_slabs([torch.empty(shape, dtype=dtype) for _ in range(w)], offset)
    for o in outs:
        o.view(torch.uint8).fill_(0xFF)
    return outs


def _noalloc(xs, outs, shape, mode, chunked, E, stream):
    w, B, S, H, D = shape
    return _lib.ulysses_a2a_run_noalloc([t.data_ptr() for t in xs], [o.data_ptr() for o in outs],
                                        B, S, H, D, w, mode, chunked, E, stream.cuda_stream,
                                        wait=1)


@pytest.mark.parametrize("case", CASES, ids=lambda c: "w{}B{}S{}H{}D{}_{}_c{}_off{}".format(*c))
@pytest.mark.parametrize("mode", [0, 1])
def test_noalloc_matches_the_oracle_and_run_on_two_calls_in_a_row(case, mode):
    w, B, S, H, D, dtype, chunked, off, path = case
    off, out_off = _offsets(off)
    E = 2 if dtype == "bf16" else 4
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    make = normal_slabs if dtype == "bf16" else uniform_slabs
    in_shape = slab_shape(mode, w, B, S, H, D)
    out_shape = slab_shape(1 - mode, w, B, S, H, D)
    cpu1 = make(in_shape, w, dtype, seed0=40 + mode)
    cpu2 = make(in_shape, w, dtype, seed0=60 + mode)
    first, second = _device_slabs(cpu1, off), _device_slabs(cpu2, off)
    out1 = _poisoned(out_shape, first[0].dtype, w, out_off)
    out2 = _poisoned(out_shape, first[0].dtype, w, out_off)
    plan = UlyssesA2A(0, E).plan(first, mode, chunked=bool(chunked), out=out1)
    assert plan["path"] == path
    assert plan["peeled"] == (0 if not (off or out_off) or path != VEC else (1 if off == out_off else 2))

    # expected outputs: the CPU oracle, and the regular entry point
    oracle1 = oracle.ulysses_a2a(cpu1, mode)
    oracle2 = oracle.ulysses_a2a(cpu2, mode)
    with UlyssesA2A(0, E) as a2a:
        # the regular entry point on outputs at the same offset (same path)
        ref1, ref2 = (_poisoned(out_shape, first[0].dtype, w, out_off) for _ in range(2))
        run1 = a2a.run(first, mode, chunked=bool(chunked), out=ref1)
        run2 = a2a.run(second, mode, chunked=bool(chunked), out=ref2)
        a2a.status()

    torch.cuda.synchronize()
    rc, msg = _noalloc(first, out1, (w, B, S, H, D), mode, chunked, E, stream)
    assert rc == _lib.OK, msg
    # the second call must not allocate device memory (nor reuse stale records)
    free_before = torch.cuda.mem_get_info()[0]
    torch_before = torch.cuda.memory_allocated()
    rc, msg = _noalloc(second, out2, (w, B, S, H, D), mode, chunked, E, stream)
    assert rc == _lib.OK, msg
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before
    assert torch.cuda.memory_allocated() == torch_before
    dt = INT_OF[E]
    for k in range(w):
        got1, got2 = out1[k].cpu().view(dt), out2[k].cpu().view(dt)
        assert torch.equal(got1, oracle1[k].view(dt)), f"first call vs oracle, rank {k}"
        assert torch.equal(got2, oracle2[k].view(dt)), f"second call vs oracle, rank {k}"
        assert torch.equal(got1, run1[k].cpu().view(dt)), f"first call vs run, rank {k}"
        assert torch.equal(got2, run2[k].cpu().view(dt)), f"second call vs run, rank {k}"


def test_noalloc_rejects_more_tma_planes_than_status_records():
    # planes of just over 64 MiB (the TMA path takes launches above that): a
    # chunked call over 65 of them needs 65 status records
    w, B, S, H, D = 2, 65, 4100, 32, 128
    stream = torch.cuda.current_stream()
    xs = [torch.randint(-30000, 30000, (B, S, H, D), dtype=torch.int16, device="cuda")
          .view(torch.bfloat16) for _ in range(w)]
    outs = [torch.zeros((B, S * w, H // w, D), dtype=torch.bfloat16, device="cuda") for _ in range(w)]
    rc, msg = _noalloc(xs, outs, (w, B, S, H, D), 0, 1, 2, stream)
    assert rc == _lib.ERR_UNSUPPORTED
    assert "64" in msg and "planes" in msg
    torch.cuda.synchronize()
    assert all(int(o.view(torch.int16).abs().sum()) == 0 for o in outs), \
        "a rejected call must launch nothing"
    # the same data unchunked needs one record and is accepted; every plane is
    # re-laid out on its own, so planes 0 and 64 are checked against the oracle
    rc, msg = _noalloc(xs, outs, (w, B, S, H, D), 0, 0, 2, stream)
    assert rc == _lib.OK, msg
    for b in (0, B - 1):
        want = oracle.ulysses_a2a([t[b:b + 1].cpu() for t in xs], 0)
        for o, e in zip(outs, want):
            assert torch.equal(o[b:b + 1].cpu().view(torch.int16), e.view(torch.int16)), b
    del xs, outs
    torch.cuda.empty_cache()


@pytest.mark.parametrize("shape", [(2, 65, 3, 2, 3), (16, 65, 3, 16, 64)],
                         ids=["staged_6B_runs", "vec_w16"])
def test_noalloc_chunked_non_tma_paths_need_no_status_record(shape):
    # 65 planes, 65 launches: the staged and vector kernels keep no status record
    w, B, S, H, D = shape
    stream = torch.cuda.current_stream()
    cpu = normal_slabs((B, S, H, D), w, "bf16", seed0=90)
    xs = [t.cuda() for t in cpu]
    outs = [torch.full((B, S * w, H // w, D), float("nan"), dtype=torch.bfloat16, device="cuda")
            for _ in range(w)]
    rc, msg = _noalloc(xs, outs, (w, B, S, H, D), 0, 1, 2, stream)
    assert rc == _lib.OK, msg
    want = oracle.ulysses_a2a(cpu, 0)
    assert all(torch.equal(o.cpu().view(torch.int16), e.view(torch.int16)) for o, e in zip(outs, want))


def test_noalloc_rejects_bad_arguments_with_a_message():
    stream = torch.cuda.current_stream()
    xs = [t.cuda() for t in normal_slabs((1, 4, 4, 8), 2, "bf16")]
    outs = [torch.zeros((1, 8, 2, 8), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    rc, msg = _lib.ulysses_a2a_run_noalloc([t.data_ptr() for t in xs], [xs[0].data_ptr(),
                                           outs[1].data_ptr()], 1, 4, 4, 8, 2, 0, 0, 2,
                                           stream.cuda_stream)
    assert rc == _lib.ERR_OVERLAP and "overlaps" in msg
    host = [torch.zeros((1, 8, 2, 8), dtype=torch.bfloat16) for _ in range(2)]
    rc, msg = _lib.ulysses_a2a_run_noalloc([t.data_ptr() for t in xs], [h.data_ptr() for h in host],
                                           1, 4, 4, 8, 2, 0, 0, 2, stream.cuda_stream)
    assert rc == _lib.ERR_DEVICE and msg
