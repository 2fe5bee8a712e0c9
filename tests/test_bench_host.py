"""Host-side logic of bench.py, without a GPU: how the timed step quantizes dY
for each recipe (the policy qfp4_linear_bwd follows), when the committed
DRAM-traffic figure of the GEMM may be reported, the roofline arithmetic and
the quantizer sweep's case list."""
import hashlib
import json
import os
import shutil

import pytest

import bench
import helpers
from fp4_precision_b200 import qfp4 as Q


def cfgs(name):
    r = Q.recipe(name)
    return r.fprop, r.dgrad, r.wgrad


@pytest.mark.parametrize("name,fused,dual", [
    ("QUARTET2_NVFP4", True, False),   # same 16-point Hadamard: one amax pass; Quartet II keeps two passes
    ("NVIDIA_NVFP4", False, False),    # different Hadamards, SR: neither
    ("AMD_MXFP4_H", False, True),      # MXFP4 (no amax), round to nearest: one read for both
])
def test_dy_plan_of_the_presets(name, fused, dual):
    assert bench.dy_plan(Q, cfgs(name), 16384) == (fused, dual)


def test_dy_plan_of_custom_recipes():
    r = Q.recipe("QUARTET2_NVFP4")
    c = [r.fprop, r.dgrad, r.wgrad]
    for g in c[1:]:
        g.rnd_a = g.rnd_b = Q.RTN
    assert bench.dy_plan(Q, c, 16384) == (True, True)       # NVFP4 RTN, same Hadamard
    c[1].had = Q.HAD_NONE
    assert bench.dy_plan(Q, c, 16384) == (False, True)      # row none, column 16: still one read
    c[1].had = Q.HAD_DET32
    assert bench.dy_plan(Q, c, 16384) == (False, False)     # a row Hadamard of another size
    c[1].had = Q.HAD_RAND16
    assert bench.dy_plan(Q, c, 16384 + 32) == (True, False)  # tokens not a multiple of 64


@pytest.mark.parametrize("name,plan", [
    ("QUARTET2_NVFP4", (True, True)),   # NVFP4 in all three GEMMs: X and W amaxes from the forward's read
    ("NVIDIA_NVFP4", (True, True)),
    ("AMD_MXFP4_H", (False, False)),    # MXFP4 has no tensor amax
])
def test_xw_plan_of_the_presets(name, plan):
    assert bench.xw_plan(Q, cfgs(name)) == plan


def test_xw_plan_needs_nvfp4_on_both_gemms():
    r = Q.recipe("QUARTET2_NVFP4")
    c = [r.fprop, r.dgrad, r.wgrad]
    c[2].fmt = Q.MXFP4
    assert bench.xw_plan(Q, c) == (False, True)    # X's backward operand is MXFP4
    c[2].fmt, c[1].fmt = Q.NVFP4, Q.MXFP4
    assert bench.xw_plan(Q, c) == (True, False)


def test_traffic_is_reported_only_for_the_profiled_sources(monkeypatch):
    root = helpers.scratch_dir("bench_root_")
    try:
        csrc = os.path.join(root, "fp4_precision_b200", "csrc")
        os.makedirs(csrc)
        os.makedirs(os.path.join(root, "profiles"))
        for f, text in (("gemm_sm100.cu", "// gemm\n"), ("qfp4_device.cuh", "// header\n")):
            with open(os.path.join(csrc, f), "w") as fh:
                fh.write(text)
        h = {f: hashlib.sha256(open(os.path.join(csrc, f), "rb").read()).hexdigest()
             for f in ("gemm_sm100.cu", "qfp4_device.cuh")}
        rec = os.path.join(root, "profiles", "gemm_traffic.json")
        with open(rec, "w") as fh:
            json.dump({"traffic_bytes_per_launch": {"fprop": 100, "dgrad": 200, "wgrad": 300},
                       "source_sha256": h}, fh)
        monkeypatch.setattr(bench, "ROOT", root)
        assert bench.measured_gemm_traffic() == {"fprop": 100, "dgrad": 200, "wgrad": 300}
        with open(os.path.join(csrc, "qfp4_device.cuh"), "a") as fh:
            fh.write("// changed\n")
        assert bench.measured_gemm_traffic() is None
        os.remove(rec)
        assert bench.measured_gemm_traffic() is None
    finally:
        shutil.rmtree(root, ignore_errors=True)


def test_roofline_follows_the_timed_region_and_the_clock():
    """The GEMM roofline uses the burst bf16 peak (x 4) for a short timed
    region and the sustained one for a region of a second or more; the
    clock-normalised fraction is the flops per SM and sampled cycle over the
    FP4 MMA's per-cycle work."""
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    flops = [1e12, 1e12, 1e12]
    ms = [0.5, 0.5, 0.5]  # 2000 TFLOP/s
    clocks = {"sm_mhz": 1500.0}
    short = bench.gemm_roofline(flops, ms, peaks, "measured", clocks, 148, 100.0)
    assert short["achieved"] == 2000.0 and short["peak"] == 6400.0 and short["frac"] == 0.3125
    long = bench.gemm_roofline(flops, ms, peaks, "measured", clocks, 148, 2500.0)
    assert long["peak"] == 5600.0
    per_cycle = 2000e12 / (148 * 1500e6)
    assert abs(long["clock_normalised"]["frac"] - per_cycle / bench.FP4_FLOP_PER_SM_CYCLE) < 1e-4
    assert bench.FP4_FLOP_PER_SM_CYCLE == 32768
    assert "clock_normalised" not in bench.gemm_roofline(flops, ms, peaks, "measured", {"sm_mhz": None}, 148, 1.0)


def test_sweep_covers_every_case():
    cases = bench.sweep_cases()
    assert len(cases) == 90 and len({c[0] for c in cases}) == 90
    assert sum(1 for c in cases if c[1] != 2) == 60  # NVFP4 and MXFP4; the rest are the round-up variant
