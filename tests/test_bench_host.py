"""Host-side logic of bench.py, without a GPU: how the timed step quantizes dY
for each recipe (the policy qfp4_linear_bwd follows), and when the committed
DRAM-traffic figure of the GEMM may be reported."""
import hashlib
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


def _profile_text(gemm_hash, header_hash):
    return ("traffic_bytes_per_launch fprop=100 dgrad=200 wgrad=300\n"
            f"gemm_source_sha256 {gemm_hash}\ndevice_header_sha256 {header_hash}\n")


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
        prof = os.path.join(root, "profiles", "gemm_bs_fp4_mlp_up.md")
        with open(prof, "w") as fh:
            fh.write(_profile_text(h["gemm_sm100.cu"], h["qfp4_device.cuh"]))
        monkeypatch.setattr(bench, "ROOT", root)
        assert bench.measured_gemm_traffic() == {"fprop": 100, "dgrad": 200, "wgrad": 300}
        with open(os.path.join(csrc, "qfp4_device.cuh"), "a") as fh:
            fh.write("// changed\n")
        assert bench.measured_gemm_traffic() is None
        os.remove(prof)
        assert bench.measured_gemm_traffic() is None
    finally:
        shutil.rmtree(root, ignore_errors=True)
