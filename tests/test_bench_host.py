"""Host arithmetic of bench.py (CPU): the layer roofline's algorithmic flops
and bytes against hand-worked figures, the clock summary of an nvidia-smi
capture, and the rule that stale DRAM counters are not reported."""
import json
import os
import sys

import pytest

import moe_inputs as mi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


# F = 2 T k 3 H I (+ 2 T 3 H I_s), B = 3 H I x 2 bytes per active expert
# + x + y + router weights (+ shared expert), worked out by hand.
HAND = {
    # 2*4096*2*3*4096*14336 ; 8 experts: 8*3*4096*14336*2 + 2*4096*4096*2 + 8*4096*2
    "mixtral_8x7b_layer": (2886.218022912e9, 8, 2818572288 + 67108864 + 65536),
    # 2*8192*4*3*2880*2880 ; 32 experts: 32*3*2880*2880*2 + 2*8192*2880*2 + 32*2880*2
    "gpt_oss_20b_layer": (1630.7453952e9, 32, 1592524800 + 94371840 + 184320),
    # 2*16384*8*3*7168*2048 + 2*16384*3*7168*2048 ; 256 experts + shared
    "fine_grained_e256_layer": (12987.981103104e9, 256,
                                22548578304 + 469762048 + 3670016 + 88080384),
    # 2*32768*8*3*2048*768 ; 128 experts
    "qwen3_30b_a3b_layer": (2473.901162496e9, 128, 1207959552 + 268435456 + 524288),
}


@pytest.mark.parametrize("name", sorted(HAND))
def test_layer_flops_and_bytes_match_hand_worked_figures(name):
    wl = mi.FULL[name]
    F, active, B = HAND[name]
    assert bench.layer_flops(wl) == pytest.approx(F, rel=1e-12)
    assert bench.layer_bytes(wl, active) == pytest.approx(B, rel=1e-12)


def test_decode_bytes_count_only_the_active_experts():
    wl = mi.FULL["gpt_oss_20b_layer"].with_(T=1)
    # 4 experts x 3 x 2880^2 x 2 bytes = 199 MB of weights, + x, y and the router
    assert bench.layer_bytes(wl, 4) == 4 * 3 * 2880 * 2880 * 2 + 2 * 2880 * 2 + 32 * 2880 * 2


def _summary(tmp_path, lines):
    s = bench.ClockSampler(None)
    s.path = str(tmp_path / "clocks.csv")
    with open(s.path, "w") as f:
        f.write("".join(line + "\n" for line in lines))
    return s.summary()


def test_clock_summary_median_max_and_reasons(tmp_path):
    rows = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1500, 1965, 999.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1400, 1965, 998.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "garbage line",
    ]
    s = _summary(tmp_path, rows)
    assert s["sm_mhz"] == 1500 and s["sm_max_mhz"] == 1965 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"] and s["power_w_max"] == 999.0
    hot = _summary(tmp_path, ["0, 1200, 1965, 800, 0x48, Not Active, Active, Not Active, Not Active"])
    assert hot["reasons"] == ["hw_thermal_slowdown"]


def test_clock_summary_without_samples_says_so(tmp_path):
    assert _summary(tmp_path, [])["reasons"] == ["unsampled"]


def test_traffic_is_reported_only_for_the_profiled_source():
    d = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for kernel, rec in d.items():
        wl = mi.FULL[rec["workload"]].with_(T=rec["T"])
        got = bench.traffic_for(kernel, wl)
        assert got is None or got == float(rec["dram_bytes_per_launch"])
        # another token count is another launch: no counters for it
        assert bench.traffic_for(kernel, wl.with_(T=rec["T"] + 1)) is None
    assert bench.traffic_for("no_such_kernel", mi.FULL["mixtral_8x7b_layer"]) is None
