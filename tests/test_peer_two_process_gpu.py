"""PeerExchange across two processes (gloo group, both on cuda:0), vs the oracle.

Each process is one rank: it builds its window, exports it, and maps the other
process's window through CUDA IPC (the path two GPUs take; here both windows
sit on the same device). The barriers are host barriers (stream synchronise +
gloo barrier), so no kernel of one process waits for the other's. Expected
values come from the oracle, computed in each process on the seeded inputs of
both ranks.
"""

import os
from datetime import timedelta

import pytest

pytestmark = pytest.mark.gpu

CASES = [
    # ((B, S_local, H, D), chunked)
    ((2, 37, 8, 64), False),
    ((2, 37, 8, 64), True),
    ((1, 512, 16, 128), False),     # larger: the windows grow (close + rebuild)
    ((3, 19, 4, 13), True),         # odd D: narrow vectors
]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist

    import oracle
    from sequence_all_re_b200.peer import PeerExchange
    from synth import normal_slabs

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    report = {"rank": rank, "ok": [], "grew": [], "error": None}
    try:
        torch.cuda.set_device(0)
        ex = PeerExchange(device=0, elem_bytes=2)
        assert ex.barrier_kind == "host"
        for shape, chunked in CASES:
            xs = normal_slabs(shape, world, "bf16")
            want_y = oracle.ulysses_a2a(xs, 0)[rank]
            y = ex.all_to_all_4d(xs[rank].cuda(), 0, chunked=chunked)
            z = ex.all_to_all_4d(y, 1, chunked=chunked)
            torch.cuda.synchronize()
            report["ok"].append(torch.equal(y.cpu().view(torch.int16), want_y.view(torch.int16)) and
                                torch.equal(z.cpu().view(torch.int16), xs[rank].view(torch.int16)))
            report["grew"].append(ex._nbytes)
        # in place: the slab is written straight into this rank's window
        shape = (1, 512, 16, 128)
        xs = normal_slabs(shape, world, "bf16", seed0=4321)
        n0 = ex.native.launch_count
        buf = ex.input_buffer(shape, torch.bfloat16)
        own = ex.native.window(rank)
        assert buf.data_ptr() in (own, own + ex._nbytes // 2)   # one of the two halves
        buf.copy_(xs[rank].cuda())
        y = ex.all_to_all_4d(buf, 0)
        del buf
        torch.cuda.synchronize()
        report["in_place_ok"] = torch.equal(y.cpu().view(torch.int16),
                                            oracle.ulysses_a2a(xs, 0)[rank].view(torch.int16))
        report["in_place_launches"] = ex.native.launch_count - n0
        # q, k, v packed: one barrier per direction
        T = 3
        shape = (2, 37, T, 8, 64)
        packed = normal_slabs(shape, world, "bf16", seed0=555)
        flat = [t.reshape(-1) for t in packed]
        outs = ex.all_to_all_4d_packed(packed[rank].cuda(), 0)
        ok = True
        for t in range(T):
            want = oracle.ulysses_a2a_pitched(flat, 0, world, 2, 37, 8, 64, T * 8 * 64,
                                              offset=t * 8 * 64)[rank]
            ok = ok and torch.equal(outs[t].cpu().reshape(-1).view(torch.int16),
                                    want.view(torch.int16))
        back = ex.all_to_all_4d_packed(outs, 1)
        torch.cuda.synchronize()
        report["packed_ok"] = ok and torch.equal(back.cpu().view(torch.int16),
                                                 packed[rank].view(torch.int16))
        # autograd: the backward of a mode-0 exchange is the mode-1 exchange
        from sequence_all_re_b200.autograd import peer_all_to_all_4d
        from synth import uniform_slabs
        shape = (2, 37, 8, 64)
        xs = normal_slabs(shape, world, "bf16", seed0=99)
        gys = uniform_slabs((2, 37 * world, 8 // world, 64), world, "bf16", seed0=7)
        x = xs[rank].cuda().requires_grad_()
        y = peer_all_to_all_4d(ex, x, 0)
        y.backward(gys[rank].cuda())
        torch.cuda.synchronize()
        report["grad_ok"] = torch.equal(x.grad.cpu().view(torch.int16),
                                        oracle.ulysses_a2a(gys, 1)[rank].view(torch.int16))
        n1 = ex.native.launch_count
        report["closed"] = ex.close()
        report["launches"] = n1
        ex.native.close()
    except Exception as e:  # reported to the parent, which fails the test
        report["error"] = repr(e)
    finally:
        q.put(report)
        dist.destroy_process_group()


def test_two_processes_exchange_through_ipc_windows():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 31000 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    reports = []
    for _ in procs:
        reports.append(q.get(timeout=300))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rep in sorted(reports, key=lambda r: r["rank"]):
        assert rep["error"] is None, rep
        assert all(rep["ok"]), rep
        assert rep["closed"] is True
        # windows: two halves of one plane when chunked, of the whole slab
        # otherwise; grown once for the large case, never shrunk
        assert rep["grew"] == [2 * (2 * 37 * 8 * 64 * 2)] * 2 + [2 * (512 * 16 * 128 * 2)] * 2
        # publish + pull per exchange (per plane when chunked), two exchanges per case,
        # then one in-place exchange: a pull and nothing else
        assert rep["in_place_ok"] is True and rep["in_place_launches"] == 1
        assert rep["grad_ok"] is True and rep["packed_ok"] is True
        # ... a packed exchange each way (1 + 1 then 3 + 1 launches: one pull for all three tensors), and a forward +
        # backward exchange of publish + pull each
        assert rep["launches"] == 2 * 2 * (1 + 2 + 1 + 3) + 1 + (1 + 1) + (3 + 1) + 2 * 2
