"""qfp4_linear_fwd_noalloc: the forward pass for callers that cannot allocate
device memory (a memory plan fixed at start-up, an allocator owned by a host
framework, or a path where cudaMalloc's possible device synchronisation is not
acceptable). It runs the same kernels as qfp4_linear_fwd with the library's
fixed 32 MiB scratch in place of a caller workspace, so its output must equal
the workspace entry point's bit for bit (stricter than the GEMM bound the other
tests use), call after call, whatever an earlier call left in the scratch.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import pytest
import torch

from fp4_precision_b200 import inputs
from fp4_precision_b200 import qfp4 as Q

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    wl = inputs.workload("tiny")
    X, W = wl["X"].cuda(), wl["W"].cuda()
    X2 = inputs.normal((384, 512), 1.0, 31, "X2").cuda()
    W2 = inputs.normal((256, 512), 0.02, 31, "W2").cuda()
    cases = [
        (X, W, Q.recipe("QUARTET2_NVFP4"), Q.make_seed(11, 12)),
        (X2, W2, Q.recipe("AMD_MXFP4_H"), Q.make_seed(13, 14)),
        (X, W, Q.recipe("NVIDIA_NVFP4"), Q.make_seed(15, 16)),
    ]
    for Xc, Wc, rec, seed in cases:
        ref = Q.linear_fwd(Xc, Wc, rec, seed)  # existing entry point, caller workspace
        Q.status()
        for _ in range(2):  # two calls in a row on the shared scratch
            got = Q.linear_fwd_noalloc(Xc, Wc, rec, seed)
            Q.status()
            assert torch.equal(got, ref)


def test_noalloc_rejects_layers_beyond_the_scratch():
    rec = Q.recipe("QUARTET2_NVFP4")
    seed = Q.make_seed(1, 2)
    M = N = K = 8192  # workspace ~ 70 MB > 32 MiB
    assert Q.linear_workspace_bytes(False, M, N, K, rec) > Q.NOALLOC_SCRATCH_BYTES
    dummy = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    status = Q.lib().qfp4_linear_fwd_noalloc(p, p, p, M, N, K, ctypes.byref(rec), ctypes.byref(seed),
                                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert status == Q.ERR_TOO_LARGE
    assert b"32 MiB" in Q.lib().qfp4_strerror(status)
    Q.status()
