"""Multi-process host logic of bench.py on CPU (gloo, world size 2; no GPU).

Each GPU of a multi-GPU run holds its own independent instance of the
re-layout (all w logical ranks of one instance live in that GPU's memory), so
the only cross-rank step is the timing: the job's time is the slowest rank's,
and its throughput counts every rank's bytes.
"""

import json
import os
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [70.0, 95.5][rank]
        slowest = bench.max_over_ranks(local_ms, dist, "cpu")
        value = bench.job_gbs(world, 2 * 201326592, 100, slowest)
        dist.barrier()
        out_q.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, slowest, value in got:
        assert slowest == 95.5                       # every rank sees the slowest time
        assert abs(value - 2 * 2 * 201326592 * 100 / 0.0955 / 1e9) < 1e-6


def test_single_rank_identity():
    assert bench.max_over_ranks(12.5) == 12.5
    assert abs(bench.job_gbs(1, 10**9, 1, 1000.0) - 1.0) < 1e-12


def _bench(args, env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], env=env,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_nonzero_rank_exits_quietly():
    r = _bench(["--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "0"],
               {"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_line():
    r = _bench(["--impl", "reference", "--gpus", "2", "--steps", "2", "--warmup", "1"],
               {"RANK": "0", "LOCAL_RANK": "0", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 2
    assert d["unit"] == "GB/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def _exchange_worker(rank, world, port, out_q):
    import oracle
    from synth import normal_slabs

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = []
        for (B, S, H, D) in ((2, 5, 4, 8), (1, 7, 6, 3)):
            xs = normal_slabs((B, S, H, D), world, "fp32", seed0=40)
            y = bench.nccl_all_to_all_4d(xs[rank], 0)
            z = bench.nccl_all_to_all_4d(y, 1)
            res.append(torch.equal(y, oracle.ulysses_a2a(xs, 0)[rank]) and torch.equal(z, xs[rank]))
        out_q.put((rank, res))
    finally:
        dist.destroy_process_group()


def test_library_all_to_all_comparison_arm_matches_the_oracle_gloo():
    """bench.py --exchange nccl's all-to-all arm, run here over gloo on CPU
    tensors: the same element map as the oracle, and mode 1 undoes mode 0."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 33500 + os.getpid() % 500
    procs = [ctx.Process(target=_exchange_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == [(0, [True, True]), (1, [True, True])]


def _bench_exchange_worker(rank, world, port, out_q):
    from test_peer_cpu import ShmNative

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = dict(w=world, B=1, S_local=6, H=4, D=8)
        res = bench.exchange_arms(dist, torch.device("cpu"), rank, world, steps=3, warmup=1, wl=wl,
                                  native=ShmNative(rank))
        out_q.put((rank, bench.exchange_keys(res)))
    except BaseException as e:          # report, so the parent does not wait for nothing
        out_q.put((rank, repr(e)))
    finally:
        dist.destroy_process_group()


def test_multi_gpu_bench_line_carries_both_exchange_arms_gloo():
    """bench.py's multi-GPU exchange section (run_ours with N > 1 ranks) on CPU
    gloo ranks, with host windows standing in for the peer object: the round
    trip holds on every rank (checked inside), and the line gets
    exchange_peer_gbs, exchange_nccl_gbs and the barrier share."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 34100 + os.getpid() % 500
    procs = [ctx.Process(target=_bench_exchange_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=240) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in (0, 1):
        keys = got[rank]
        assert isinstance(keys, dict), keys
        ex = keys["exchange"]
        # a few-KB slab on CPU: GB/s rounds to ~0, the step times are what count
        assert keys["exchange_peer_gbs"] == ex["peer"]["gbs"] >= 0
        assert keys["exchange_nccl_gbs"] == ex["nccl"]["gbs"] >= 0
        assert ex["peer"]["ms_per_step"] > 0 and ex["nccl"]["ms_per_step"] > 0
        assert ex["peer"]["barriers_per_step"] == 2 and 0 < ex["peer"]["barrier_share"]
        assert ex["steps"] == 3 and "w = 2" in ex["workload"]
    # both ranks report the same (max-over-ranks) times
    assert got[0]["exchange"]["peer"]["ms_per_step"] == got[1]["exchange"]["peer"]["ms_per_step"]
