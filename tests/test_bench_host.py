"""Host-side consistency of bench.py, without a GPU: every workload names a
synthetic layer that exists, pruned workloads keep fewer experts than their
layer has, the algorithmic FLOP count matches the expert maths, and the
committed launch-list summary of the default workload is found (its DRAM
traffic is reported while the kernel sources match the recorded hash, and
null after a change)."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from bit_expert_gemm_b200 import synth  # noqa: E402


def test_workload_table():
    for name, (wname, T, kind) in bench.WORKLOADS.items():
        wl = synth.WORKLOADS[wname]
        assert kind in ("forward", "refill"), name
        assert T >= 1 and wl.H % 64 == 0 and wl.I % 64 == 0, name
    for name, keep in bench.PRUNED.items():
        wname, T, kind = bench.WORKLOADS[name]
        assert kind == "forward" and 0 < keep < synth.WORKLOADS[wname].E
    assert bench.WORKLOADS["bf16_prefill"] == ("bf16", 8192, "forward")


def test_expert_flops_and_default_traffic():
    # gate, up and down of one routed row: 2 * 3 * H * I FLOP
    assert bench.expert_flops(81920, 2048, 640) == 2.0 * 81920 * 3 * 2048 * 640
    traffic, src = bench.measured_traffic("bf16_prefill")
    assert src is not None and "moe_layer_bf16_prefill_t8192.md" in src
    assert traffic is None or traffic > 2e9  # the expert call moves at least the touched experts' 2.1 GB
    assert bench.measured_traffic("no_such_workload") == (None, None)


def test_clock_record_rules():
    # hardware or thermal slowdowns reject the timed region; a power cap alone is kept
    ok = {"sm_mhz": 1965.0, "sm_max_mhz": 1965, "reasons": []}
    assert not bench.clocks_rejected(ok)
    assert not bench.clocks_rejected({**ok, "sm_mhz": 1335.0, "reasons": ["sw_power_cap"]})
    for r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"):
        assert bench.clocks_rejected({**ok, "reasons": [r]})
        assert bench.clocks_rejected({**ok, "reasons": ["sw_power_cap", r]})
    # clocks well below the maximum with no reason: a clock lock left on the GPU
    assert bench.clocks_rejected({**ok, "sm_mhz": 1200.0})
    assert not bench.clocks_rejected({**ok, "sm_mhz": 1900.0})
    # no NVML: nothing to judge
    assert not bench.clocks_rejected({"sm_mhz": None, "sm_max_mhz": None, "reasons": ["NVML unavailable: x"]})


def test_every_traffic_line_names_existing_sources():
    # each committed traffic line parses, names kernel sources that exist, and
    # is found by measured_traffic for its workload (a renamed source would
    # otherwise turn the figure into a silent null)
    import glob
    import re
    pat = re.compile(r"traffic: workload=(\S+) bytes_per_launch=(\d+) sources=(\S+) sha256=([0-9a-f]+)")
    seen = set()
    for path in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        for line in open(path):
            m = pat.search(line)
            if not m:
                continue
            wk, nbytes, srcs = m.group(1), int(m.group(2)), m.group(3).split(",")
            assert wk in bench.WORKLOADS, wk
            assert nbytes > 0
            for f in srcs:
                assert os.path.isfile(os.path.join(ROOT, "bit_expert_gemm_b200", "csrc", f)), (path, f)
            assert bench.measured_traffic(wk)[1] is not None
            seen.add(wk)
    assert {"bf16_prefill", "bf16_decode_t1", "awq_decode_t1", "awq_prefill", "nvfp4_prefill",
            "nvfp4_decode_t1"} <= seen


def test_workload_labels():
    # both arms name a workload with the same label; pruned workloads state the kept expert count
    for name, (wname, T, kind) in bench.WORKLOADS.items():
        label = bench.workload_label(name)
        assert label.startswith(f"{name}: T={T} ")
        assert ("Refill-RMS accumulate" in label) == (kind == "refill")
    for name, keep in bench.PRUNED.items():
        assert f" E={keep} " in bench.workload_label(name)
    assert bench.workload_label("bf16_prefill") == "bf16_prefill: T=8192 H=2048 E=512 k=10 I=640 shared=640 fmt=bf16"
