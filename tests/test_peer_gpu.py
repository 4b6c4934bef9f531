"""The multi-GPU exchange entry points (ulysses_a2a_peer_*) vs the CPU oracle.

All w ranks live in this one process on cuda:0: each rank has its own library
context and window, the records are exchanged in memory, and every kernel runs
on one stream in the order publish (every rank), then pull (every rank), which
is the order the caller's barriers give on separate GPUs. No kernel waits for
another. Outputs are poisoned and guarded as in test_parity_gpu.py; expected
values come from the oracle only.
"""

import pytest
import torch

import oracle
from sequence_all_re_b200 import UlyssesA2A, _lib, mode0_local_tuple
from synth import normal_slabs, uniform_slabs, unique_slabs

from test_parity_gpu import Guarded, bits

pytestmark = pytest.mark.gpu


class LocalRanks:
    """w ranks of the exchange in this process, one context and window each."""

    def __init__(self, w, E, nbytes):
        self.w = w
        self.ctxs = [UlyssesA2A(0, E) for _ in range(w)]
        self.peers, self.records = [], []
        for k in range(w):
            rc, h, rec = _lib.ulysses_a2a_peer_create(self.ctxs[k]._ctx, k, w, nbytes)
            assert rc == _lib.OK, self.ctxs[k].last_error()
            self.peers.append(h)
            self.records.append(rec)

    def open(self):
        for k in range(self.w):
            rc = _lib.ulysses_a2a_peer_open(self.peers[k], self.records)
            assert rc == _lib.OK, self.ctxs[k].last_error()
        return self

    def launches(self):
        return sum(c.launch_count for c in self.ctxs)

    def exchange(self, xs, outs, mode, chunked=False, in_pitch=0, out_pitch=0):
        """Publish every rank's slab, then pull every rank's output (per plane if chunked)."""
        stream = torch.cuda.current_stream().cuda_stream
        B, S, H, D = mode0_local_tuple(tuple(xs[0].shape), mode, self.w)
        planes = range(B) if chunked else [None]
        nb = 1 if chunked else B
        for b in planes:
            for k in range(self.w):
                x = xs[k] if b is None else xs[k][b:b + 1]
                rc = _lib.ulysses_a2a_peer_publish(self.peers[k], x.data_ptr(), nb, S, H, D, mode,
                                                   in_pitch, stream)
                assert rc == _lib.OK, self.ctxs[k].last_error()
            for k in range(self.w):
                o = outs[k] if b is None else outs[k][b:b + 1]
                rc = _lib.ulysses_a2a_peer_pull(self.peers[k], o.data_ptr(), nb, S, H, D, mode,
                                                out_pitch, stream)
                assert rc == _lib.OK, self.ctxs[k].last_error()
        torch.cuda.synchronize()

    def close(self):
        for p in self.peers:
            assert _lib.ulysses_a2a_peer_close(p) == _lib.OK
        for p in self.peers:
            assert _lib.ulysses_a2a_peer_destroy(p) == _lib.OK
        for c in self.ctxs:
            c.close()


def slab_bytes(shape, E):
    n = E
    for v in shape:
        n *= v
    return n


CASES = [
    # (w, B, S_local, H, D)
    (1, 1, 33, 4, 64),
    (2, 3, 37, 4, 64),
    (4, 2, 100, 8, 128),
    (8, 2, 53, 40, 128),
    (3, 2, 29, 6, 32),
    (8, 1, 7, 8, 256),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "w{}B{}S{}H{}D{}".format(*c))
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("chunked", [False, True], ids=["whole", "per_plane"])
def test_peer_exchange_matches_oracle(case, mode, chunked):
    w, B, S, H, D = case
    xs0 = normal_slabs((B, S, H, D), w, "bf16")
    xs_cpu = xs0 if mode == 0 else oracle.ulysses_a2a(xs0, 0)
    want = oracle.ulysses_a2a(xs_cpu, mode)
    nbytes = slab_bytes(xs_cpu[0].shape, 2) // (B if chunked else 1)
    ranks = LocalRanks(w, 2, nbytes).open()
    try:
        xs = [t.cuda() for t in xs_cpu]
        g = Guarded(tuple(want[0].shape), torch.bfloat16, w)
        before = ranks.launches()
        ranks.exchange(xs, g.slabs, mode, chunked=chunked)
        # one publish and one pull launch per rank (per plane when chunked)
        assert ranks.launches() - before == 2 * w * (B if chunked else 1)
        for k in range(w):
            assert torch.equal(bits(g.slabs[k].cpu()), bits(want[k])), f"rank {k}"
        g.check_guards()
    finally:
        ranks.close()


def test_peer_round_trip_reuses_the_windows():
    w, B, S, H, D = 4, 2, 300, 16, 64
    xs_cpu = unique_slabs((B, S, H, D), w, 4)      # every element traceable
    ranks = LocalRanks(w, 4, slab_bytes((B, S, H, D), 4)).open()
    try:
        xs = [t.cuda() for t in xs_cpu]
        ys = [torch.empty(B, S * w, H // w, D, dtype=torch.int32, device="cuda") for _ in range(w)]
        zs = [torch.empty_like(x) for x in xs]
        for _ in range(3):
            ranks.exchange(xs, ys, 0)
            ranks.exchange(ys, zs, 1)
        want = oracle.ulysses_a2a(xs_cpu, 0)
        for k in range(w):
            assert torch.equal(ys[k].cpu(), want[k])
            assert torch.equal(zs[k].cpu(), xs_cpu[k])
    finally:
        ranks.close()


def test_peer_fp32_and_narrow_vectors():
    # D*E = 2 * 13 bytes per run: the pull takes 2-byte vectors
    for dtype, E, shape in ((torch.float32, 4, (2, 41, 8, 32)), (torch.bfloat16, 2, (1, 19, 4, 13))):
        w = 4
        xs_cpu = uniform_slabs(shape, w, "fp32" if E == 4 else "bf16")
        ranks = LocalRanks(w, E, slab_bytes(shape, E)).open()
        try:
            xs = [t.cuda() for t in xs_cpu]
            want = oracle.ulysses_a2a(xs_cpu, 0)
            g = Guarded(tuple(want[0].shape), dtype, w)
            ranks.exchange(xs, g.slabs, 0)
            for k in range(w):
                assert torch.equal(bits(g.slabs[k].cpu()), bits(want[k]))
            g.check_guards()
        finally:
            ranks.close()


def test_peer_packed_qkv_in_and_out():
    """mode 0 publishes q straight out of a packed [B, S, 3, H, D] buffer; mode 1
    pulls into the k slot of another packed buffer, leaving q and v untouched."""
    w, B, S, H, D = 4, 2, 45, 8, 64
    packed_cpu = normal_slabs((B, S, 3, H, D), w, "bf16")
    q_cpu = [p[:, :, 0].contiguous() for p in packed_cpu]
    ranks = LocalRanks(w, 2, slab_bytes((B, S, H, D), 2)).open()
    try:
        packed = [p.cuda() for p in packed_cpu]
        ys = [torch.empty(B, S * w, H // w, D, dtype=torch.bfloat16, device="cuda")
              for _ in range(w)]
        ranks.exchange([p[:, :, 0] for p in packed], ys, 0, in_pitch=3 * H * D)
        want = oracle.ulysses_a2a(q_cpu, 0)
        for k in range(w):
            assert torch.equal(bits(ys[k].cpu()), bits(want[k]))
        dst = [torch.full((B, S, 3, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
               for _ in range(w)]
        ranks.exchange(ys, [d[:, :, 1] for d in dst], 1, out_pitch=3 * H * D)
        for k in range(w):
            got = dst[k].cpu()
            assert torch.equal(bits(got[:, :, 1]), bits(q_cpu[k]))
            assert bool(torch.isnan(got[:, :, 0].float()).all())
            assert bool(torch.isnan(got[:, :, 2].float()).all())
    finally:
        ranks.close()


def test_one_pull_writes_only_its_own_output():
    w, B, S, H, D = 4, 1, 64, 8, 64
    xs_cpu = normal_slabs((B, S, H, D), w, "bf16")
    ranks = LocalRanks(w, 2, slab_bytes((B, S, H, D), 2)).open()
    try:
        xs = [t.cuda() for t in xs_cpu]
        stream = torch.cuda.current_stream().cuda_stream
        for k in range(w):
            assert _lib.ulysses_a2a_peer_publish(ranks.peers[k], xs[k].data_ptr(), B, S, H, D, 0,
                                                 0, stream) == _lib.OK
        want = oracle.ulysses_a2a(xs_cpu, 0)
        g = Guarded(tuple(want[0].shape), torch.bfloat16, w)
        assert _lib.ulysses_a2a_peer_pull(ranks.peers[2], g.slabs[2].data_ptr(), B, S, H, D, 0, 0,
                                          stream) == _lib.OK
        torch.cuda.synchronize()
        assert torch.equal(bits(g.slabs[2].cpu()), bits(want[2]))
        for k in (0, 1, 3):
            assert bool((g.slabs[k].view(torch.int16) == -1).all()), "another rank's output was written"
        g.check_guards()
    finally:
        ranks.close()


def test_peer_errors_launch_nothing():
    w, B, S, H, D = 2, 1, 64, 4, 64
    nbytes = slab_bytes((B, S, H, D), 2)
    stream = torch.cuda.current_stream().cuda_stream
    x = torch.zeros(B, S, H, D, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(B, S * w, H // w, D, dtype=torch.bfloat16, device="cuda")
    ranks = LocalRanks(w, 2, nbytes)
    try:
        p0, c0 = ranks.peers[0], ranks.ctxs[0]
        n0 = ranks.launches()
        # pull before the windows are open
        assert _lib.ulysses_a2a_peer_pull(p0, out.data_ptr(), B, S, H, D, 0, 0, stream) == _lib.ERR_INVALID
        assert "not open" in c0.last_error()
        # records out of rank order, corrupted, or from another world size
        swapped = [ranks.records[1], ranks.records[0]]
        assert _lib.ulysses_a2a_peer_open(p0, swapped) == _lib.ERR_INVALID
        bad = bytearray(ranks.records[1])
        bad[0] ^= 0xFF
        assert _lib.ulysses_a2a_peer_open(p0, [ranks.records[0], bytes(bad)]) == _lib.ERR_INVALID
        rc, h3, rec3 = _lib.ulysses_a2a_peer_create(ranks.ctxs[1]._ctx, 1, 3, nbytes)
        assert rc == _lib.OK
        assert _lib.ulysses_a2a_peer_open(p0, [ranks.records[0], rec3]) == _lib.ERR_INVALID
        assert _lib.ulysses_a2a_peer_destroy(h3) == _lib.OK
        ranks.open()
        assert _lib.ulysses_a2a_peer_open(p0, ranks.records) == _lib.ERR_INVALID  # already open
        # a slab larger than the window
        big = torch.zeros(2, S, H, D, dtype=torch.bfloat16, device="cuda")
        assert _lib.ulysses_a2a_peer_publish(p0, big.data_ptr(), 2, S, H, D, 0, 0, stream) == _lib.ERR_INVALID
        assert "exceeds the window" in c0.last_error()
        # H not divisible by the world size; a pitched mode-1 input; a pitched mode-0 output
        assert _lib.ulysses_a2a_peer_publish(p0, x.data_ptr(), B, S, 3, D, 0, 0, stream) == _lib.ERR_INVALID
        assert _lib.ulysses_a2a_peer_publish(p0, out.data_ptr(), B, S, H, D, 1, 2 * H * D,
                                             stream) == _lib.ERR_INVALID
        assert _lib.ulysses_a2a_peer_pull(p0, out.data_ptr(), B, S, H, D, 0, 2 * H * D,
                                          stream) == _lib.ERR_INVALID
        # an output that overlaps a window (here the peer's, as mapped in this process)
        win1 = _lib.ulysses_a2a_peer_window(p0, 1)
        assert win1 != 0 and _lib.ulysses_a2a_peer_window(p0, 2) == 0
        assert _lib.ulysses_a2a_peer_window_bytes(p0) == nbytes
        assert _lib.ulysses_a2a_peer_pull(p0, win1, B, S, H, D, 0, 0, stream) == _lib.ERR_OVERLAP
        # an input that is not device memory
        host = torch.zeros(B, S, H, D, dtype=torch.bfloat16)
        assert _lib.ulysses_a2a_peer_publish(p0, host.data_ptr(), B, S, H, D, 0, 0,
                                             stream) == _lib.ERR_DEVICE
        # empty calls succeed without a launch
        assert _lib.ulysses_a2a_peer_publish(p0, 0, 0, S, H, D, 0, 0, stream) == _lib.OK
        assert _lib.ulysses_a2a_peer_pull(p0, 0, B, 0, H, D, 0, 0, stream) == _lib.OK
        assert ranks.launches() == n0
        # bad arguments to create
        assert _lib.ulysses_a2a_peer_create(c0._ctx, 2, 2, nbytes)[0] == _lib.ERR_INVALID
        assert _lib.ulysses_a2a_peer_create(c0._ctx, 0, 65, nbytes)[0] == _lib.ERR_INVALID
        assert _lib.ulysses_a2a_peer_create(c0._ctx, 0, 2, 0)[0] == _lib.ERR_INVALID
        # the context still runs a correct exchange after every rejection
        xs_cpu = normal_slabs((B, S, H, D), w, "bf16")
        want = oracle.ulysses_a2a(xs_cpu, 0)
        outs = [torch.empty_like(out) for _ in range(w)]
        ranks.exchange([t.cuda() for t in xs_cpu], outs, 0)
        for k in range(w):
            assert torch.equal(bits(outs[k].cpu()), bits(want[k]))
    finally:
        ranks.close()


def test_publishing_the_own_window_copies_nothing():
    """Zero-copy publish: a slab already in the rank's own window is left in place."""
    w, B, S, H, D = 4, 2, 33, 8, 64
    xs_cpu = normal_slabs((B, S, H, D), w, "bf16")
    ranks = LocalRanks(w, 2, slab_bytes((B, S, H, D), 2)).open()
    try:
        stream = torch.cuda.current_stream().cuda_stream
        xs = [t.cuda() for t in xs_cpu]
        for k in range(w):      # an ordinary publish puts each slab into its window
            assert _lib.ulysses_a2a_peer_publish(ranks.peers[k], xs[k].data_ptr(), B, S, H, D, 0, 0,
                                                 stream) == _lib.OK
        n0 = ranks.launches()
        for k in range(w):
            own = _lib.ulysses_a2a_peer_window(ranks.peers[k], k)
            assert _lib.ulysses_a2a_peer_publish(ranks.peers[k], own, B, S, H, D, 0, 0,
                                                 stream) == _lib.OK
            # the window as a pitched source is not in place: it overlaps the window
            assert _lib.ulysses_a2a_peer_publish(ranks.peers[k], own, B, S, H, D, 0, 2 * H * D,
                                                 stream) == _lib.ERR_OVERLAP
        assert ranks.launches() == n0
        want = oracle.ulysses_a2a(xs_cpu, 0)
        g = Guarded(tuple(want[0].shape), torch.bfloat16, w)
        for k in range(w):
            assert _lib.ulysses_a2a_peer_pull(ranks.peers[k], g.slabs[k].data_ptr(), B, S, H, D, 0,
                                              0, stream) == _lib.OK
        torch.cuda.synchronize()
        for k in range(w):
            assert torch.equal(bits(g.slabs[k].cpu()), bits(want[k]))
        g.check_guards()
    finally:
        ranks.close()


def test_packed_exchange_through_window_offsets():
    """q, k, v packed per rank: one publish of the packed slab and a pull per tensor
    (windows read with row pitch T*H*D at the tensor's head offset); back in mode 1
    with the T slabs at consecutive window offsets, pulled into the packed slots."""
    T, w, B, S, H, D = 3, 4, 2, 37, 8, 64
    E = 2
    slab = B * S * H * D * E
    packed_cpu = normal_slabs((B, S, T, H, D), w, "bf16", seed0=880)
    flat = [t.reshape(-1) for t in packed_cpu]
    ranks = LocalRanks(w, E, T * slab).open()
    try:
        stream = torch.cuda.current_stream().cuda_stream
        packed = [t.cuda() for t in packed_cpu]
        n0 = ranks.launches()
        for k in range(w):
            assert _lib.ulysses_a2a_peer_publish(ranks.peers[k], packed[k].data_ptr(), B, S, T * H,
                                                 D, 0, 0, stream) == _lib.OK
        outs = [[torch.empty(B, S * w, H // w, D, dtype=torch.bfloat16, device="cuda")
                 for _ in range(T)] for _ in range(w)]
        for k in range(w):
            for t in range(T):
                rc = _lib.ulysses_a2a_peer_pull(ranks.peers[k], outs[k][t].data_ptr(), B, S, H, D, 0,
                                                T * H * D, stream, window_offset=t * H * D * E)
                assert rc == _lib.OK, ranks.ctxs[k].last_error()
        torch.cuda.synchronize()
        assert ranks.launches() - n0 == w + w * T
        for t in range(T):
            want = oracle.ulysses_a2a_pitched(flat, 0, w, B, S, H, D, T * H * D, offset=t * H * D)
            for k in range(w):
                assert torch.equal(bits(outs[k][t].cpu()).reshape(-1), bits(want[k])), (t, k)
        # mode 1: rank k's T slabs at window offsets t*slab, pulled into packed slots
        for k in range(w):
            for t in range(T):
                assert _lib.ulysses_a2a_peer_publish(ranks.peers[k], outs[k][t].data_ptr(), B, S, H,
                                                     D, 1, 0, stream, window_offset=t * slab) == _lib.OK
        back = [torch.full((B, S, T, H, D), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
                for _ in range(w)]
        for k in range(w):
            for t in range(T):
                rc = _lib.ulysses_a2a_peer_pull(ranks.peers[k], back[k][:, :, t].data_ptr(), B, S, H,
                                                D, 1, T * H * D, stream, window_offset=t * slab)
                assert rc == _lib.OK, ranks.ctxs[k].last_error()
        torch.cuda.synchronize()
        for k in range(w):
            assert torch.equal(bits(back[k].cpu()), bits(packed_cpu[k])), k
        # offsets: not a multiple of the element size, past the window, or leaving too
        # little room for the slab
        p0 = ranks.peers[0]
        n1 = ranks.launches()
        assert _lib.ulysses_a2a_peer_publish(p0, packed[0].data_ptr(), B, S, H, D, 0, T * H * D,
                                             stream, window_offset=1) == _lib.ERR_INVALID
        assert _lib.ulysses_a2a_peer_pull(p0, outs[0][0].data_ptr(), B, S, H, D, 0, T * H * D,
                                          stream, window_offset=T * slab + 2) == _lib.ERR_INVALID
        assert _lib.ulysses_a2a_peer_publish(p0, outs[0][0].data_ptr(), B, S, H, D, 1, 0, stream,
                                             window_offset=T * slab - slab // 2) == _lib.ERR_INVALID
        assert _lib.ulysses_a2a_peer_pull(p0, outs[0][0].data_ptr(), B, S, H, D, 0, T * H * D,
                                          stream, window_offset=T * H * D * E) == _lib.ERR_INVALID
        assert ranks.launches() == n1
    finally:
        ranks.close()


def test_packed_exchange_pulls_every_tensor_in_one_launch():
    """ulysses_a2a_peer_pull_packed: mode 0 pulls rank k's head group of all T
    tensors from the packed windows in one launch; mode 1 pulls the T gathered
    slabs (at window offsets t*slab) into rank k's packed slab in one launch.
    Same bytes as T pitched oracle calls; ragged S_local and odd D (narrow
    vectors) included."""
    E = 2
    for (T, w, B, S, H, D) in ((3, 4, 2, 37, 8, 64), (2, 2, 1, 19, 4, 13), (3, 8, 1, 11, 40, 128)):
        slab = B * S * H * D * E
        packed_cpu = normal_slabs((B, S, T, H, D), w, "bf16", seed0=890 + T + w)
        flat = [t.reshape(-1) for t in packed_cpu]
        ranks = LocalRanks(w, E, T * slab).open()
        try:
            stream = torch.cuda.current_stream().cuda_stream
            packed = [t.cuda() for t in packed_cpu]
            for k in range(w):
                assert _lib.ulysses_a2a_peer_publish(ranks.peers[k], packed[k].data_ptr(), B, S,
                                                     T * H, D, 0, 0, stream) == _lib.OK
            outs = [[torch.full((B, S * w, H // w, D), -1, dtype=torch.int16, device="cuda")
                     .view(torch.bfloat16) for _ in range(T)] for _ in range(w)]
            n0 = ranks.launches()
            for k in range(w):
                rc = _lib.ulysses_a2a_peer_pull_packed(ranks.peers[k],
                                                       [o.data_ptr() for o in outs[k]], T, B, S,
                                                       H, D, 0, stream)
                assert rc == _lib.OK, ranks.ctxs[k].last_error()
            torch.cuda.synchronize()
            assert ranks.launches() - n0 == w            # one launch per rank for all T
            for t in range(T):
                want = oracle.ulysses_a2a_pitched(flat, 0, w, B, S, H, D, T * H * D,
                                                  offset=t * H * D)
                for k in range(w):
                    assert torch.equal(bits(outs[k][t].cpu()).reshape(-1), bits(want[k])), (t, k)
            for k in range(w):
                for t in range(T):
                    assert _lib.ulysses_a2a_peer_publish(ranks.peers[k], outs[k][t].data_ptr(), B,
                                                         S, H, D, 1, 0, stream,
                                                         window_offset=t * slab) == _lib.OK
            back = [torch.full((B, S, T, H, D), -1, dtype=torch.int16, device="cuda")
                    .view(torch.bfloat16) for _ in range(w)]
            n1 = ranks.launches()
            for k in range(w):
                rc = _lib.ulysses_a2a_peer_pull_packed(ranks.peers[k], [back[k].data_ptr()], T, B,
                                                       S, H, D, 1, stream)
                assert rc == _lib.OK, ranks.ctxs[k].last_error()
            torch.cuda.synchronize()
            assert ranks.launches() - n1 == w
            for k in range(w):
                assert torch.equal(bits(back[k].cpu()), bits(packed_cpu[k])), k
            # too many tensors for the windows, or T * w above the limit: rejected, nothing launched
            n2 = ranks.launches()
            assert _lib.ulysses_a2a_peer_pull_packed(ranks.peers[0], [back[0].data_ptr()], T + 1, B,
                                                     S, H, D, 1, stream) == _lib.ERR_INVALID
            assert _lib.ulysses_a2a_peer_pull_packed(ranks.peers[0], [back[0].data_ptr()], 65, B,
                                                     S, H, D, 1, stream) == _lib.ERR_INVALID
            assert ranks.launches() == n2
        finally:
            ranks.close()
