"""bench.py's host-side arithmetic, checked without a GPU: the algorithmic bytes and flops of the
layer (the closed forms of the roofline), the kernel count a forward launches, the roofline fractions
formed from stage times, and the rule that a captured DRAM-traffic figure is reported only while the
kernel sources it was captured from are unchanged."""
import os
import shutil

import pytest

import bench
import beam_synth as bs


def test_layer_bytes_and_flops_closed_forms():
    # per active expert: three 2560 x 5120 bf16 matrices; W_r fp32; x in and y out bf16; ids + weights
    wl = bs.get("prefill")
    a = bench.algorithmic(wl, 256)
    assert a["layer_bytes"] == 256 * 78_643_200 + 5_242_880 + 4096 * 20_544  # the roofline's closed form
    assert a["layer_bytes"] == 256 * 3 * 2560 * 5120 * 2 + 256 * 5120 * 4 + 2 * 4096 * 5120 * 2 + 4096 * 8 * 8
    # per token: the router's 2 H E plus 8 experts x (gate, up, down) = 6 H I multiply-adds x 2
    assert a["layer_flops"] == 4096 * (2 * 5120 * 256 + 8 * 6 * 5120 * 2560)
    # the gate/up launch: both weight matrices of every active expert once + x in
    assert a["stage_bytes"]["gate_up_swiglu"] == 256 * 2 * 2560 * 5120 * 2 + 4096 * 5120 * 2
    assert abs(a["stage_bytes"]["gate_up_swiglu"] / 1e9 - 13.464) < 1e-3
    # an expert no token picks moves no weight bytes
    assert bench.algorithmic(wl, 248)["layer_bytes"] == a["layer_bytes"] - 8 * 3 * 2560 * 5120 * 2


def test_low_precision_weight_bytes():
    wl = bs.get("decode")
    b16 = bench.algorithmic(wl, 256)["stage_bytes"]["down"]
    assert bench.algorithmic(wl, 256, "mxfp8")["stage_bytes"]["down"] == pytest.approx(b16 / 2 * (1 + 1 / 32))
    assert bench.algorithmic(wl, 256, "w4a4")["stage_bytes"]["down"] == pytest.approx(b16 / 2 * (0.5 + 1 / 16))


@pytest.mark.parametrize("name,block,fmt,n", [
    ("prefill", False, "bf16", 5 + 6 + 1),   # screened router, dispatch, row gather, GEMMs, combine
    ("decode", False, "bf16", 1 + 6),        # direct router, narrow tiles (no row gather)
    ("prefill", True, "bf16", 5 + 6 + 1 + 1),  # + the pre-norm
    ("prefill", False, "mxfp8", 5 + 6 + 1 + 1),  # + the activation quantiser
    ("long", False, "bf16", 5 + 6 + 1),
])
def test_launches_per_step(name, block, fmt, n):
    assert bench.launches_per_step(bs.get(name), block, fmt) == n


def test_roofline_fractions_from_stage_times():
    wl = bs.get("prefill")
    pk = dict(bench.FALLBACK_PEAKS)
    a = bench.algorithmic(wl, 256)
    stage_ms = {"router": 0.25, "dispatch": 0.02, "gather": 0.07, "gate_up_swiglu": 2.2, "down": 1.25,
                "combine": 0.12}
    ms_step = sum(stage_ms.values())
    layer, roof = bench.roofline_of(wl, "bf16", stage_ms, 256, ms_step, pk, "fallback")
    assert layer["bound"] == "hbm"
    assert layer["roofline_ms"] == pytest.approx(a["layer_bytes"] / (pk["hbm_gbs"] * 1e9) * 1e3)
    assert layer["frac"] == pytest.approx(layer["roofline_ms"] / ms_step)
    # the dominant launch is gate/up, HBM-bound at prefill: its bytes over its time over the copy peak
    assert roof["kernel"] == "gate_up_swiglu" and roof["bound"] == "hbm"
    assert roof["achieved"] == pytest.approx(a["stage_bytes"]["gate_up_swiglu"] / 2.2e-3 / 1e9)
    assert roof["frac"] == pytest.approx(roof["achieved"] / pk["hbm_gbs"])
    # at T=65536 the products dominate: tensor-bound against the sustained bf16 peak
    wl = bs.get("long")
    stage_ms = dict(stage_ms, gate_up_swiglu=26.0, down=17.0)
    _, roof = bench.roofline_of(wl, "bf16", stage_ms, 256, sum(stage_ms.values()), pk, "fallback")
    assert roof["bound"] == "tensor" and roof["peak"] == pk["bf16_tflops_sustained"]
    assert roof["achieved"] == pytest.approx(bench.algorithmic(wl, 256)["stage_flops"]["gate_up_swiglu"] / 26e-3 / 1e12)


def test_traffic_reported_only_for_the_captured_sources(tmp_path, monkeypatch):
    key = ("gate_up_swiglu", "prefill")
    entry = bench.NCU_TRAFFIC[key]
    assert bench.traffic_of(*key[:1], "bf16", key[1]) == entry["bytes"]
    assert bench.traffic_of("gate_up_swiglu", "bf16", "skew") is None  # never captured
    # a copy of the sources with one tracked file edited: the figure no longer applies
    csrc = tmp_path / "csrc"
    shutil.copytree(bench._CSRC, csrc)
    monkeypatch.setattr(bench, "_CSRC", str(csrc))
    assert bench.traffic_of("gate_up_swiglu", "bf16", "prefill") == entry["bytes"]
    with open(os.path.join(csrc, entry["files"][0]), "a") as f:
        f.write("\n// edited\n")
    assert bench.traffic_of("gate_up_swiglu", "bf16", "prefill") is None
