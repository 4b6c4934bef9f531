"""bench.py host logic without a GPU: the ncu traffic lookup and the workload table."""

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from sequence_all_re_b200 import _lib  # noqa: E402


def plan_dict(w, B, S, H, D, path=_lib.PATH_AUTO, E=2, off=0, goff=None):
    """The plan of a mode-0 call whose input slabs sit `off` bytes past 4 KiB
    boundaries and whose output slabs sit `goff` (default: `off`) bytes past."""
    goff = off if goff is None else goff
    step = (B * S * H * D * E + 4095) // 4096 * 4096 + 4096
    ins = [(1 << 40) + k * step + off for k in range(w)]
    outs = [(1 << 40) + (w + k) * step + goff for k in range(w)]
    rc, p, msg = _lib.ulysses_a2a_plan(ins, outs, B, S, H, D, w, 0, 0, E, forced_path=path)
    assert rc == _lib.OK, msg
    return p.as_dict()


def test_committed_captures_match_the_current_kernels_and_plans():
    traffic = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))["workloads"]
    for key, entry in traffic.items():
        path, shape = key.split(":")
        parts = shape.split("_")
        w, B, S, H, D = (int(part[1:]) for part in parts[:5])
        E = {"bf16": 2, "fp32": 4}[parts[5]]
        off = int(parts[6][4:]) if len(parts) > 6 else 0
        goff = int(parts[7][8:]) if len(parts) > 7 else off     # "_gathered<n>"
        # the planner chooses this kernel for the captured shape (AUTO) ...
        assert plan_dict(w, B, S, H, D, _lib.PATH_AUTO, E, off, goff)["path"] == {
            "tma": _lib.PATH_TMA, "vec": _lib.PATH_VEC, "staged": _lib.PATH_STAGED}[path] or (
            key == "vec:w4_B1_S8192_H24_D128_bf16")          # the VEC capture of a TMA shape
        # ... and the capture matches its launch shape and code
        p = plan_dict(w, B, S, H, D, {"tma": _lib.PATH_TMA, "vec": _lib.PATH_VEC,
                                      "staged": _lib.PATH_STAGED}[path], E, off, goff)
        got, why = bench.ncu_traffic(key, p, 0)
        assert why == "ncu", (key, why)
        assert got == entry["dram_bytes_per_launch"]
        # DRAM reads of a launch cover the payload (no re-reads beyond a few per mille)
        payload = w * B * S * H * D * E
        for m in ("mode0", "mode1"):
            assert 0.999 * payload <= entry[m]["dram_read"] <= 1.002 * payload, (key, m)


def test_traffic_is_withheld_when_the_launch_differs():
    wl = bench.WORKLOADS[bench.DEFAULT_WORKLOAD]
    key = bench.workload_key(wl["w"], wl["B"], wl["S_local"], wl["H"], wl["D"], "tma")
    p = plan_dict(wl["w"], wl["B"], wl["S_local"], wl["H"], wl["D"])
    assert bench.ncu_traffic(key, p, 0)[1] == "ncu"
    assert bench.ncu_traffic(key, dict(p, grid=p["grid"] + 1), 0) == (
        None, "the capture was taken with another launch shape")
    assert bench.ncu_traffic(key, p, 1)[0] is None                 # chunked launches
    assert bench.ncu_traffic("tma:w3_B1_S7_H3_D8_bf16", p, 0) == (
        None, "no ncu capture of this kernel and workload")


def test_workload_table_names_each_workload_by_its_sizes():
    for name, wl in bench.WORKLOADS.items():
        parts = {p[0]: int(p[1:]) for p in name.split("_")}
        assert parts["w"] == wl["w"] and parts["S"] == wl["S_local"]
        assert parts["H"] == wl["H"] and parts["D"] == wl["D"]
        assert parts.get("B", 1) == wl["B"]
    assert bench.DEFAULT_WORKLOAD in bench.WORKLOADS


def test_clock_windows_cover_only_their_timed_region():
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.samples = [(1.0, 1965.0, ()), (2.0, 1800.0, ("sw_power_cap",)), (3.0, 1965.0, ()),
                 (4.0, 900.0, ("hw_slowdown",))]
    s.max_mhz, s.source = 1965.0, "nvml"
    w = s.window(1.5, 3.5)
    assert w == {"sm_mhz": 1882.5, "sm_max_mhz": 1965.0, "samples": 2,
                 "reasons": ["sw_power_cap"], "source": "nvml"}
    assert s.window(4.5, 5.0) is None
    assert s.window(0.0, 9.0)["reasons"] == ["hw_slowdown", "sw_power_cap"]


def test_fractions_count_twice_the_payload():
    # 1 GB of payload in 1 ms: 1000 GB/s of payload, 2000 GB/s of traffic
    f = bench.fracs(10**9, 1.0, 4000.0)
    assert f == {"gbs": 1000.0, "frac": 0.5, "frac_nominal": 0.25}


def test_vector_shapes_are_named_by_their_sizes_and_leave_the_tma_path():
    for name, shape in bench.VEC_SHAPES.items():
        w, B, S, H, D, E, off = shape[:7]
        goff = shape[7] if len(shape) > 7 else off
        assert f"w{w}_" in name and f"S{S}_" in name and f"H{H}_" in name and f"D{D}" in name
        row = (H // w) * D * E
        tma_blocked = row % 16 != 0 or off % 16 != 0 or goff % 16 != 0 or w > 8
        assert tma_blocked, name
        wl = bench.ALL_WORKLOADS[name]
        assert (wl["off"], wl["goff"]) == (off, goff)


def test_staged_form_shapes_are_named_by_their_sizes_and_dense():
    for name, (w, B, S, H, D, E) in bench.STAGED_FORM_SHAPES.items():
        parts = {p[0]: p[1:] for p in name.split("_")}
        assert (int(parts["w"]), int(parts["S"]), int(parts["H"]), int(parts["D"])) == (w, S, H, D)
        assert ("fp32" in name) == (E == 4) and ("u8" in name) == (E == 1)
        row = (H // w) * D * E
        assert row % 16 != 0                   # TMA cannot take them
        p = plan_dict(w, B, S, H, D, _lib.PATH_STAGED, E)
        assert p["path"] == _lib.PATH_STAGED and p["fixed_phase"] == 1, name


def test_one_sided_offsets_are_keyed_apart():
    assert bench.workload_key(4, 1, 8, 24, 128, "vec", 2, 2) == "vec:w4_B1_S8_H24_D128_bf16_base2"
    assert bench.workload_key(4, 1, 8, 24, 128, "vec", 2, 2, 0) == \
        "vec:w4_B1_S8_H24_D128_bf16_base2_gathered0"
    # the bench's one-sided shape takes the shifted vector kernel in both modes
    w, B, S, H, D, E, off, goff = bench.VEC_SHAPES["base2in_w4_S8192_H24_D128"]
    p = plan_dict(w, B, S, H, D, _lib.PATH_AUTO, E, off, goff)
    assert p["path"] == _lib.PATH_VEC and p["peeled"] == 2
