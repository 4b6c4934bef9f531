"""Host logic of PeerExchange on CPU: gloo, world size 2, no GPU.

The native peer object is replaced by a stand-in whose windows are POSIX
shared memory and whose pull assembles the rank's output from the other
process's window with tensor slicing. What is under test is the sequencing
that PeerExchange owns: the record exchange, the one barrier of an exchange
(before its pull), the two window halves that exchanges use in turn, window
growth (collective close + rebuild), the agreement on call signatures, and
collective teardown. Delays make a missing barrier or a reused half visible.
Rank 1 publishes late, so rank 0, pulling without the barrier, would read rank
1's window before it is written; rank 1 also pulls late, so rank 0,
publishing its next exchanges into the same half, would overwrite it while
rank 1 still reads it. Expected values come from the oracle.
"""

import os
import time
from datetime import timedelta
from multiprocessing import shared_memory

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


class _HostStream:
    def synchronize(self):
        pass


class ShmNative:
    """Stand-in for sequence_all_re_b200.peer.NativePeer with host windows."""

    def __init__(self, rank, publish_delay=0.0, pull_delay=0.0, fail_create=False):
        self.device = torch.device("cpu")
        self.elem_bytes = 2
        self.rank = rank
        self.world = None
        self.own = None
        self.peers = {}
        self.log = []
        self.publish_delay = publish_delay
        self.pull_delay = pull_delay
        self.fail_create = fail_create
        self.launch_count = 0
        self.halves = []           # the window offset of every pull

    def create(self, rank, world, nbytes):
        if self.fail_create:
            raise RuntimeError("window allocation failed (injected)")
        self.world = world
        self.own = shared_memory.SharedMemory(create=True, size=nbytes)
        self.log.append(("create", nbytes))
        return self.own.name

    def open(self, records):
        for k, name in enumerate(records):
            if k != self.rank:
                self.peers[k] = shared_memory.SharedMemory(name=name)
        self.log.append(("open",))

    def _win(self, k, dtype, shape, offset_bytes=0, strides=None):
        """Rank k's window as a tensor of `shape` from byte offset_bytes on
        (dense, or with the given element strides)."""
        shm = self.own if k == self.rank else self.peers[k]
        esz = torch.empty((), dtype=dtype).element_size()
        whole = torch.frombuffer(shm.buf, dtype=dtype, count=shm.size // esz)
        if strides is None:
            strides = []
            acc = 1
            for v in reversed(shape):
                strides.insert(0, acc)
                acc *= v
        return whole.as_strided(tuple(shape), tuple(strides), offset_bytes // esz)

    def window(self, rank):
        shm = self.own if rank == self.rank else self.peers.get(rank)
        if shm is None:
            return 0
        return torch.frombuffer(shm.buf, dtype=torch.uint8, count=1).data_ptr()

    def window_tensor(self, shape, dtype, offset=0):
        n = 1
        for v in shape:
            n *= v
        return torch.frombuffer(self.own.buf, dtype=dtype, count=n, offset=offset).view(shape)

    def publish(self, x, B, S, H, D, mode, row_pitch, stream, window_offset=0):
        time.sleep(self.publish_delay)
        w = self.world
        shape = (B, S, H, D) if mode == 0 else (B, S * w, H // w, D)
        src = x if tuple(x.shape) == shape else x.reshape(shape)   # a packed slab: T*H heads
        self._win(self.rank, x.dtype, shape, window_offset).copy_(src)
        self.log.append("publish")

    def pull(self, out, B, S, H, D, mode, row_pitch, stream, window_offset=0):
        time.sleep(self.pull_delay)
        self.halves.append(window_offset)
        w, k = self.world, self.rank
        Hw = H // w
        if mode == 0:
            p = row_pitch or H * D                 # the windows' row pitch
            o = out.view(B, w, S, Hw, D)
            for j in range(w):
                win = self._win(j, out.dtype, (B, S, H, D), window_offset, (S * p, p, D, 1))
                o[:, j] = win[:, :, k * Hw:(k + 1) * Hw]
        else:
            for r in range(w):
                win = self._win(r, out.dtype, (B, S * w, Hw, D), window_offset)
                out[:, :, r * Hw:(r + 1) * Hw] = win[:, k * S:(k + 1) * S]
        self.log.append("pull")

    def pull_packed(self, outs, T, B, S, H, D, mode, stream, window_offset=0):
        """The T tensors of a head-packed exchange at once (one native launch)."""
        time.sleep(self.pull_delay)
        self.halves.append(window_offset)
        w, k = self.world, self.rank
        Hw = H // w
        slab_bytes = B * S * H * D * self.elem_bytes
        if mode == 0:
            for t in range(T):
                o = outs[t].view(B, w, S, Hw, D)
                for j in range(w):
                    win = self._win(j, o.dtype, (B, S, T, H, D), window_offset)
                    o[:, j] = win[:, :, t, k * Hw:(k + 1) * Hw]
        else:
            for t in range(T):
                for r in range(w):
                    win = self._win(r, outs.dtype, (B, S * w, Hw, D), window_offset + t * slab_bytes)
                    outs[:, :, t, r * Hw:(r + 1) * Hw] = win[:, k * S:(k + 1) * S]
        self.log.append("pull")

    def unmap(self):
        for shm in self.peers.values():
            shm.close()
        self.peers.clear()
        self.log.append(("unmap",))

    def release(self):
        if self.own is not None:
            self.own.close()
            self.own.unlink()
            self.own = None
            self.log.append(("release",))

    def abandon(self):
        self.log.append(("abandon",))
        self.own = None            # left to the process's exit, never unlinked here
        self.peers = {}

    def current_stream(self):
        return _HostStream()

    def synchronize(self):
        pass

    def close(self):
        self.release()


def _worker(rank, world, port, scenario, q):
    import oracle
    from sequence_all_re_b200.peer import PeerExchange
    from synth import normal_slabs, uniform_slabs

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    rep = {"rank": rank, "ok": [], "errors": []}
    try:
        if scenario == "exchange":
            # rank 0 never waits; rank 1 publishes late and pulls late
            native = ShmNative(rank, publish_delay=0.05 if rank == 1 else 0.0,
                               pull_delay=0.2 if rank == 1 else 0.0)
            ex = PeerExchange(native=native, elem_bytes=2)
            calls = [((2, 5, 4, 8), 0, False, normal_slabs),
                     ((2, 5, 4, 8), 0, False, uniform_slabs),   # same size: windows reused
                     ((2, 5, 4, 8), 1, True, normal_slabs),
                     ((1, 16, 8, 8), 0, False, uniform_slabs)]  # larger: grow
            for shape, mode, chunked, gen in calls:
                xs = gen(shape, world, "bf16")
                if mode == 0:
                    x, want = xs[rank], oracle.ulysses_a2a(xs, 0)[rank]
                else:
                    x, want = oracle.ulysses_a2a(xs, 0)[rank], xs[rank]
                got = ex.all_to_all_4d(x, mode, chunked=chunked)
                rep["ok"].append(torch.equal(got.view(torch.int16), want.view(torch.int16)))
            rep["closed"] = ex.close()
            rep["log"] = native.log
            rep["halves"] = native.halves
        elif scenario == "in_place":
            # rank 1 writes its slab late and pulls late: input_buffer() hands
            # out the half no rank reads any more (rank 0 writing into the half
            # rank 1 still reads would show); without the barrier before the
            # pull, rank 0 would read rank 1's window before the slab is in it
            native = ShmNative(rank, pull_delay=0.2 if rank == 1 else 0.0)
            ex = PeerExchange(native=native, elem_bytes=2)
            shape = (2, 5, 4, 8)
            for it in range(3):
                xs = normal_slabs(shape, world, "bf16", seed0=1000 + 10 * it)
                buf = ex.input_buffer(shape, torch.bfloat16)
                if rank == 1:
                    time.sleep(0.05)
                buf.copy_(xs[rank])
                got = ex.all_to_all_4d(buf, 0)
                del buf
                want = oracle.ulysses_a2a(xs, 0)[rank]
                rep["ok"].append(torch.equal(got.view(torch.int16), want.view(torch.int16)))
            # an ordinary call still works after in-place ones, also after an
            # input_buffer() that no exchange used (its half is taken again)
            for seed in (2000, 2010):
                if seed == 2010:
                    ex.input_buffer(shape, torch.bfloat16)
                xs = normal_slabs(shape, world, "bf16", seed0=seed)
                got = ex.all_to_all_4d(xs[rank].clone(), 0)
                rep["ok"].append(torch.equal(got.view(torch.int16),
                                             oracle.ulysses_a2a(xs, 0)[rank].view(torch.int16)))
            rep["halves"] = native.halves
            rep["closed"] = ex.close()
            rep["log"] = native.log
        elif scenario == "autograd":
            from sequence_all_re_b200.autograd import peer_all_to_all_4d
            ex = PeerExchange(native=ShmNative(rank), elem_bytes=2)
            shape = (2, 5, 4, 8)
            xs = normal_slabs(shape, world, "bf16")
            gys = uniform_slabs((2, 5 * world, 4 // world, 8), world, "bf16", seed0=77)
            x = xs[rank].clone().requires_grad_()
            y = peer_all_to_all_4d(ex, x, 0)
            y.backward(gys[rank])
            # forward: mode 0 of the rank slabs; backward: mode 1 of the gradients
            rep["ok"].append(torch.equal(y.detach().view(torch.int16),
                                         oracle.ulysses_a2a(xs, 0)[rank].view(torch.int16)))
            rep["ok"].append(torch.equal(x.grad.view(torch.int16),
                                         oracle.ulysses_a2a(gys, 1)[rank].view(torch.int16)))
            rep["closed"] = ex.close()
        elif scenario == "packed":
            # q, k, v packed per rank: one publish and one pull in mode 0; T
            # publishes at window offsets and one pull into the packed slots in mode 1
            native = ShmNative(rank, publish_delay=0.05 if rank == 1 else 0.0,
                               pull_delay=0.2 if rank == 1 else 0.0)
            ex = PeerExchange(native=native, elem_bytes=2)
            T, B, S, H, D = 3, 2, 5, 4, 8
            packed = normal_slabs((B, S, T, H, D), world, "bf16", seed0=600)
            flat = [t.reshape(-1) for t in packed]
            outs = ex.all_to_all_4d_packed(packed[rank], 0)
            for t in range(T):
                want = oracle.ulysses_a2a_pitched(flat, 0, world, B, S, H, D, T * H * D,
                                                  offset=t * H * D)[rank]
                rep["ok"].append(torch.equal(outs[t].reshape(-1).view(torch.int16),
                                             want.view(torch.int16)))
            back = ex.all_to_all_4d_packed(outs, 1)
            rep["ok"].append(torch.equal(back.view(torch.int16), packed[rank].view(torch.int16)))
            rep["closed"] = ex.close()
            rep["log"] = native.log
            rep["halves"] = native.halves
        elif scenario == "split_close":
            # rank 1 believes its window is gone while rank 0's is armed
            native = ShmNative(rank)
            ex = PeerExchange(native=native, elem_bytes=2)
            ex.all_to_all_4d(normal_slabs((1, 4, 2, 8), world, "bf16")[rank], 0)
            if rank == 1:
                ex._armed = False
            rep["closed"] = ex.close()
            rep["disabled"] = ex.disabled_reason
            rep["log"] = native.log
            try:
                ex.all_to_all_4d(torch.zeros(1, 4, 2, 8, dtype=torch.bfloat16), 0)
            except RuntimeError as e:
                rep["errors"].append(str(e))
        elif scenario == "fail_build":
            native = ShmNative(rank, fail_create=(rank == 1))
            ex = PeerExchange(native=native, elem_bytes=2)
            try:
                ex.all_to_all_4d(torch.zeros(1, 4, 2, 8, dtype=torch.bfloat16), 0)
            except RuntimeError as e:
                rep["errors"].append(str(e))
            rep["disabled"] = ex.disabled_reason
            rep["closed"] = ex.close()
            rep["log"] = native.log
        elif scenario == "mismatch":
            ex = PeerExchange(native=ShmNative(rank), elem_bytes=2)
            S = 4 if rank == 0 else 6
            try:
                ex.all_to_all_4d(torch.zeros(1, S, 2, 8, dtype=torch.bfloat16), 0)
            except ValueError as e:
                rep["errors"].append(str(e))
            rep["closed"] = ex.close()
    except Exception as e:
        rep["errors"].append("unexpected: " + repr(e))
    finally:
        q.put(rep)
        dist.destroy_process_group()


def _run(scenario, port_offset):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 32000 + port_offset + os.getpid() % 500
    procs = [ctx.Process(target=_worker, args=(r, 2, port, scenario, q)) for r in range(2)]
    for p in procs:
        p.start()
    reps = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(reps, key=lambda r: r["rank"])


def test_exchange_sequence_barriers_and_growth():
    for rep in _run("exchange", 0):
        assert rep["errors"] == [], rep
        assert rep["ok"] == [True] * 4, rep
        assert rep["closed"] is True
        log = rep["log"]
        creates = [e[1] for e in log if isinstance(e, tuple) and e[0] == "create"]
        # two halves of 2*5*4*8*2 = 640 bytes (256-byte aligned: 768) for the
        # first three calls (one plane when chunked fits), then two of the
        # larger slab's 2048 after a collective close
        assert creates == [2 * 768, 2 * 2048]
        ops = [e for e in log if isinstance(e, str)]
        # one publish + one pull per exchange, per plane when chunked
        assert ops == ["publish", "pull"] * (1 + 1 + 2 + 1)
        # the exchanges (planes, when chunked) alternate between the two
        # halves, from the first after each build
        assert rep["halves"] == [0, 768, 0, 768, 0]
        assert log.index(("unmap",)) < log.index(("release",))


def test_in_place_input_skips_the_publish():
    for rep in _run("in_place", 300):
        assert rep["errors"] == [], rep
        assert rep["ok"] == [True] * 5, rep
        assert rep["closed"] is True
        ops = [e for e in rep["log"] if isinstance(e, str)]
        # three in-place exchanges pull without publishing, then two ordinary ones
        assert ops == ["pull"] * 3 + ["publish", "pull"] * 2
        # halves 0, 1, 0 in place; then 1; the unused input_buffer() takes 0,
        # which the next exchange takes again
        assert rep["halves"] == [0, 768, 0, 768, 0], rep["halves"]


def test_autograd_backward_is_the_inverse_exchange():
    for rep in _run("autograd", 400):
        assert rep["errors"] == [], rep
        assert rep["ok"] == [True, True], rep
        assert rep["closed"] is True


def test_packed_exchange_uses_one_barrier_and_one_pull():
    for rep in _run("packed", 500):
        assert rep["errors"] == [], rep
        assert rep["ok"] == [True] * 4, rep
        assert rep["closed"] is True
        ops = [e for e in rep["log"] if isinstance(e, str)]
        # one pull (one native launch) for the three tensors in each mode, the
        # two exchanges in the two halves (T*B*S*H*D*2 = 1920 bytes, 256-byte
        # aligned: 2048)
        assert ops == ["publish", "pull"] + ["publish"] * 3 + ["pull"]
        assert rep["halves"] == [0, 2048]


def test_split_teardown_leaks_instead_of_freeing():
    for rep in _run("split_close", 600):
        assert rep["closed"] is False and "disagreed" in rep["disabled"], rep
        # the armed rank leaves its window to the process exit: no unmap, no release
        if rep["rank"] == 0:
            assert ("abandon",) in rep["log"] and ("release",) not in rep["log"], rep["log"]
        assert len(rep["errors"]) == 1 and "disabled" in rep["errors"][0], rep


def test_failed_window_build_disables_every_rank():
    reps = _run("fail_build", 100)
    for rep in reps:
        assert len(rep["errors"]) == 1 and "window build failed" in rep["errors"][0], rep
        assert rep["disabled"] is not None
        assert rep["closed"] is True             # nothing left armed anywhere
    # the rank whose allocation worked released its window again
    assert ("release",) in reps[0]["log"]


def test_ranks_with_different_arguments_all_raise():
    for rep in _run("mismatch", 200):
        assert len(rep["errors"]) == 1 and "different arguments" in rep["errors"][0], rep
        assert rep["closed"] is True
