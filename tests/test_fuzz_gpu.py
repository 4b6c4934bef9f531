"""1500 seeded random calls across every path and knob vs the CPU oracle (needs a B200).

Each case draws the rank count (1..16), element size (1/2/4/8), B, S_local, H,
D, mode, chunking (per plane, through the staging window or not), a row pitch
on the [B, S_local, H, D] side, input and output base offsets past a 16-byte
boundary (independently), head-packed tensors (T = 2, 3), a forced path (or
AUTO), the tuning knobs (rows per unit, unit order, grid-stride grids, the
staged path's fixed-phase or per-piece form) and the
entry point: ``run``, a bound call, the allocation-free C entry point, or the
host-buffer call (the last two for dense, unpacked slabs).
The element map is the one the FastVideo API docs give for ``run_armed``
(device_communicators/ulysses_a2a). Expected values come from the oracle
(the pitched form for pitched and packed cases); outputs are poisoned and
fenced, gaps between pitched rows must stay untouched. A forced path that
cannot take the shape (TMA on an unaligned or packed call, the staged path on
a strided row longer than its shared memory) must be refused before any
launch.
"""

import random

import pytest
import torch

import oracle
from sequence_all_re_b200 import A2AError, PATH_AUTO, PATH_STAGED, PATH_TMA, PATH_VEC, UlyssesA2A, _lib
from synth import random_byte_slabs
from test_parity_gpu import Guarded, bits

pytestmark = pytest.mark.gpu

INT = {1: torch.uint8, 2: torch.int16, 4: torch.int32, 8: torch.int64}


def _at_offset(t, off):
    """A device copy of t starting `off` bytes into its own allocation."""
    raw = torch.empty(t.numel() * t.element_size() + off, dtype=torch.uint8, device="cuda")
    v = raw[off:].view(t.dtype).view(t.shape)
    v.copy_(t)
    return v


def _one_case(rng, case, ctxs):
    E = rng.choice([1, 2, 2, 2, 4, 8])
    w = rng.choice([1, 2, 2, 3, 4, 4, 8, 8, 16])
    H = rng.randint(1, 4) * w
    D = rng.choice([1, 2, 3, 4, 5, 7, 8, 12, 16, 24, 32, 40, 50, 64, 100, 128])
    B, S = rng.randint(1, 3), rng.randint(1, 150)
    mode = rng.randint(0, 1)
    chunked = rng.choice([0, 0, 1, 2])
    T = rng.choice([1, 1, 1, 1, 2, 3]) if chunked != 2 and 3 * w <= 64 else 1
    gap = rng.choice([0, 0, 0, 1, 2, 4, 8]) if T == 1 else 0
    off_in = rng.choice([0, 0, 0, E, 2 * E, 8, 6, 10]) % 16
    off_in -= off_in % E
    off_out = off_in if rng.random() < 0.5 else rng.choice([0, E, 2 * E, 4, 8, 14]) % 16
    off_out -= off_out % E
    path = rng.choice([PATH_AUTO, PATH_AUTO, PATH_AUTO, PATH_TMA, PATH_VEC, PATH_STAGED])
    a2a = ctxs[E]
    a2a.set_path(path)
    form = rng.choice([0, 0, 1])
    a2a.set_tuning(rows_per_tile=rng.choice([0, 0, 1, 3, 7]), order=rng.choice([-1, 0, 1]),
                   ctas_per_sm=rng.choice([0, 0, 0, 1, 3]), staged_form=form)
    dt = INT[E]
    entry = rng.choice(["run", "run", "run", "bind", "noalloc", "host"])
    if entry in ("noalloc", "host") and (T != 1 or gap or chunked == 2):
        entry = "run"
    if entry == "host":
        path = PATH_AUTO
        a2a.set_path(path)
        off_in = off_out = 0
    if entry == "noalloc":
        path = PATH_AUTO                    # the allocation-free call takes AUTO's path
    P = T * H * D + gap                     # row pitch of the [B, S, (T,) H, D] side
    n_p = (B * S - 1) * P + T * H * D
    gshape = (B, S * w, H // w, D)
    desc = f"case {case}: E={E} w={w} B={B} S={S} H={H} D={D} mode={mode} chunked={chunked} " \
           f"T={T} gap={gap} off={off_in}/{off_out} path={path} form={form} entry={entry}"

    def call(xs, m, out):
        if entry == "bind":
            return a2a.bind(xs, m, chunked=chunked, out=out)()
        if entry == "noalloc":
            rc, msg = _lib.ulysses_a2a_run_noalloc([t.data_ptr() for t in xs],
                                                   [o.data_ptr() for o in out], B, S, H, D, w, m,
                                                   chunked, E, torch.cuda.current_stream().cuda_stream,
                                                   wait=1)
            assert rc == _lib.OK, (desc, msg)
            return out
        if entry == "host":
            res = a2a.run_host([t.cpu().pin_memory() for t in xs], m, chunked=bool(chunked))
            for o, r in zip(out, res):
                o.copy_(r)
            return out
        return a2a.run(xs, m, chunked=chunked, out=out)
    try:
        if T == 1:
            bufs = [t.view(dt) for t in random_byte_slabs((n_p * E,), w, seed0=50000 + case)]
            if mode == 0:
                want = oracle.ulysses_a2a_pitched(bufs, 0, w, B, S, H, D, P)
                xs = [_at_offset(t, off_in).as_strided((B, S, H, D), (S * P, P, D, 1)) for t in bufs]
                g = Guarded(gshape, dt, w, offset=off_out)
                call(xs, 0, g.slabs)
                a2a.status()
                for r in range(w):
                    assert torch.equal(bits(g.slabs[r].cpu()).reshape(-1), bits(want[r]).reshape(-1)), \
                        (desc, r)
                g.check_guards()
            else:
                ys = [y.reshape(gshape) for y in oracle.ulysses_a2a_pitched(bufs, 0, w, B, S, H, D, P)]
                xs = [_at_offset(y, off_in) for y in ys]
                outs = [_at_offset(torch.full((n_p,), -1, dtype=dt), off_out) for _ in range(w)]
                views = [o.as_strided((B, S, H, D), (S * P, P, D, 1)) for o in outs]
                call(xs, 1, views)
                a2a.status()
                for j in range(w):
                    got = outs[j].cpu()
                    assert torch.equal(torch.as_strided(got, (B * S, H * D), (P, 1)),
                                       torch.as_strided(bufs[j], (B * S, H * D), (P, 1))), (desc, j)
                    if gap:
                        gaps = torch.as_strided(got, (B * S - 1, gap), (P, 1), H * D)
                        assert bool((gaps == -1).all()), (desc, "gap written")
        else:
            packed = [t.view(dt).view(B, S, T, H, D)
                      for t in random_byte_slabs((B * S * T * H * D * E,), w, seed0=60000 + case)]
            flat = [t.reshape(-1) for t in packed]
            wants = [oracle.ulysses_a2a_pitched(flat, 0, w, B, S, H, D, T * H * D, offset=t * H * D)
                     for t in range(T)]
            if mode == 0:
                xs = [_at_offset(t, off_in) for t in packed]
                outs = [[_at_offset(torch.full(gshape, -1, dtype=dt), off_out) for _ in range(w)]
                        for _ in range(T)]
                a2a.run_packed(xs, 0, chunked=bool(chunked), out=outs)
                a2a.status()
                for t in range(T):
                    for r in range(w):
                        assert torch.equal(outs[t][r].cpu().reshape(-1), wants[t][r].reshape(-1)), \
                            (desc, t, r)
            else:
                ins = [[_at_offset(y.reshape(gshape), off_in) for y in wants[t]] for t in range(T)]
                back = [_at_offset(torch.full((B, S, T, H, D), -1, dtype=dt), off_out)
                        for _ in range(w)]
                a2a.run_packed(ins, 1, chunked=bool(chunked), out=back)
                a2a.status()
                for j in range(w):
                    assert torch.equal(back[j].cpu(), packed[j]), (desc, j)
        return "ran"
    except A2AError as e:
        # only a forced path may be refused: TMA on a shape it cannot describe,
        # the staged path on a strided row too long for its shared memory
        assert e.code == _lib.ERR_UNSUPPORTED and (
            path == PATH_TMA or (path == PATH_STAGED and "shared memory" in str(e))), (desc, str(e))
        return "refused"


def test_random_calls_against_the_oracle():
    rng = random.Random(4711)
    ctxs = {E: UlyssesA2A(0, E) for E in (1, 2, 4, 8)}
    try:
        outcomes = [_one_case(rng, case, ctxs) for case in range(1500)]
    finally:
        for c in ctxs.values():
            c.close()
    assert outcomes.count("ran") >= 1200
