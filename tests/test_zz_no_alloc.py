"""The allocation-free entry point, ulysses_a2a_run_noalloc (needs a B200).

Some callers cannot allocate device memory (their process's device memory is
owned by another allocator under a fixed budget, or they run where cudaMalloc
is not allowed). For them the library offers one entry point that allocates
nothing: it keeps the copy kernel's status records in a static device array.
These tests call it through the C ABI and check that its output equals the
regular entry point's (bit for bit, the tolerance every test here uses) on two
calls in a row, and that it rejects a chunked call needing more status records
than the array holds. This file is named so pytest collects it last; it also
passes when run alone in a fresh process (its first call does the one-time
per-device set-up).
"""

import pytest
import torch

from sequence_all_re_b200 import UlyssesA2A, _lib
from synth import normal_slabs, slab_shape, uniform_slabs

pytestmark = pytest.mark.gpu

INT_OF = {2: torch.int16, 4: torch.int32}

CASES = [
    # (w, B, S_local, H, D, dtype, chunked)  -- TMA path unless noted
    (4, 1, 8192, 24, 128, "bf16", 0),
    (8, 2, 4725, 40, 128, "bf16", 1),
    (2, 3, 37, 4, 64, "bf16", 1),
    (4, 2, 45, 8, 128, "fp32", 0),
    (2, 2, 17, 4, 3, "bf16", 0),      # 12-byte runs: the vector path
]


def _noalloc(xs, outs, shape, mode, chunked, E, stream):
    w, B, S, H, D = shape
    return _lib.ulysses_a2a_run_noalloc([t.data_ptr() for t in xs], [o.data_ptr() for o in outs],
                                        B, S, H, D, w, mode, chunked, E, stream.cuda_stream,
                                        wait=1)


@pytest.mark.parametrize("case", CASES, ids=lambda c: "w{}B{}S{}H{}D{}_{}_c{}".format(*c))
@pytest.mark.parametrize("mode", [0, 1])
def test_noalloc_matches_run_on_two_calls_in_a_row(case, mode):
    w, B, S, H, D, dtype, chunked = case
    E = 2 if dtype == "bf16" else 4
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    make = normal_slabs if dtype == "bf16" else uniform_slabs
    in_shape = slab_shape(mode, w, B, S, H, D)
    out_shape = slab_shape(1 - mode, w, B, S, H, D)
    first = [t.cuda() for t in make(in_shape, w, dtype, seed0=40 + mode)]
    second = [t.cuda() for t in make(in_shape, w, dtype, seed0=60 + mode)]

    # expected outputs from the regular entry point
    with UlyssesA2A(0, E) as a2a:
        want1 = a2a.run(first, mode, chunked=bool(chunked))
        want2 = a2a.run(second, mode, chunked=bool(chunked))
        a2a.status()

    out1 = [torch.full(out_shape, float("nan"), dtype=first[0].dtype, device="cuda") for _ in range(w)]
    out2 = [torch.full(out_shape, float("nan"), dtype=first[0].dtype, device="cuda") for _ in range(w)]
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
        assert torch.equal(out1[k].view(dt), want1[k].view(dt)), f"first call, rank {k}"
        assert torch.equal(out2[k].view(dt), want2[k].view(dt)), f"second call, rank {k}"


def test_noalloc_rejects_more_planes_than_status_records():
    w, B, S, H, D = 2, 65, 2, 2, 8        # a chunked call over 65 planes needs 65 records
    stream = torch.cuda.current_stream()
    xs = [t.cuda() for t in normal_slabs((B, S, H, D), w, "bf16")]
    outs = [torch.zeros((B, S * w, H // w, D), dtype=torch.bfloat16, device="cuda") for _ in range(w)]
    rc, msg = _noalloc(xs, outs, (w, B, S, H, D), 0, 1, 2, stream)
    assert rc == _lib.ERR_UNSUPPORTED
    assert "64" in msg and "planes" in msg
    torch.cuda.synchronize()
    assert all(bool((o == 0).all()) for o in outs), "a rejected call must launch nothing"
    # the same data unchunked needs one record and is accepted
    rc, msg = _noalloc(xs, outs, (w, B, S, H, D), 0, 0, 2, stream)
    assert rc == _lib.OK, msg


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
