"""Every library call that touches the device opens an NVTX range named after
its entry point. A child process loads tests/nvtx_record.c as its NVTX
injection library (NVTX_INJECTION64_PATH), which writes every push and pop to
a file; the parent checks the names, the balance and the nesting."""
import os
import subprocess
import sys

import pytest

import helpers

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys, torch
sys.path.insert(0, {root!r})
from fp4_precision_b200 import qfp4 as Q
dev = torch.device("cuda", 0)
g = torch.Generator(device="cpu").manual_seed(1)
X = torch.randn((256, 512), generator=g).to(torch.bfloat16).to(dev)
W = torch.randn((384, 512), generator=g).to(torch.bfloat16).to(dev)
dY = torch.randn((256, 384), generator=g).to(torch.bfloat16).to(dev)
seed = Q.make_seed(1, 2, 3, 4)
A = Q.quantize(X, Q.NVFP4, Q.RTN, Q.HAD_RAND16, Q.ROW, seed)
B = Q.quantize(W, Q.NVFP4, Q.RTN, Q.HAD_RAND16, Q.ROW, seed)
Q.gemm(A, B, torch.bfloat16)
rec = Q.recipe("QUARTET2_NVFP4")
Q.linear_fwd(X, W, rec, seed)
Q.linear_bwd(dY, X, W, rec, seed)
Q.linear_fwd_noalloc(X, W, rec, seed)
torch.cuda.synchronize()
Q.status()
"""


def test_entry_points_open_named_ranges():
    d = helpers.scratch_dir("nvtx_")
    lib = os.path.join(d, "libnvtx_record.so")
    subprocess.check_call(["gcc", "-shared", "-fPIC", "-O1", "-I", "/usr/local/cuda/include",
                           os.path.join(ROOT, "tests", "nvtx_record.c"), "-o", lib])
    log = os.path.join(d, "nvtx.log")
    env = dict(os.environ, NVTX_INJECTION64_PATH=lib, QFP4_NVTX_LOG=log)
    subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT)], env=env, check=True, timeout=600)
    lines = open(log).read().splitlines()
    depth, max_depth, names = 0, 0, []
    for line in lines:
        if line.startswith("push "):
            depth += 1
            max_depth = max(max_depth, depth)
            names.append(line[5:])
        else:
            assert line == "pop", line
            depth -= 1
            assert depth >= 0
    assert depth == 0, "unbalanced ranges"
    lib_names = [n for n in names if n.startswith("qfp4_")]
    for n in ("qfp4_quantize", "qfp4_gemm", "qfp4_linear_fwd", "qfp4_linear_bwd", "qfp4_linear_fwd_noalloc",
              "qfp4_status"):
        assert n in lib_names, (n, sorted(set(lib_names)))
    # the no-alloc call runs qfp4_linear_fwd inside its own range
    i = lib_names.index("qfp4_linear_fwd_noalloc")
    assert lib_names[i + 1] == "qfp4_linear_fwd"
    assert max_depth >= 2
