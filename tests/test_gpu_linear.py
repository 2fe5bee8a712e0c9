"""The FP4 linear layer (Fprop, Dgrad, Wgrad through the C ABI) vs the
oracle's composition of the same quantizations and fp64 GEMMs."""
import numpy as np
import pytest
import torch

import oracle as O
from fp4_precision_b200 import inputs
from fp4_precision_b200 import qfp4 as Q

pytestmark = pytest.mark.gpu

ROT, SRS = 0x1111_2222_3333_4444, 0x5555_6666_7777_8888


def within(D_gpu, ref, bound, bf16_out):
    Dg = D_gpu.float().cpu().numpy().astype(np.float64)
    tol = bound + (2.0 ** -8 * np.abs(ref) if bf16_out else 0.0)
    err = np.abs(Dg - ref)
    assert np.all(err <= tol), f"{np.sum(err > tol)} of {err.size} out of bound"


@pytest.mark.parametrize("preset", ["QUARTET2_NVFP4", "NVIDIA_NVFP4", "AMD_MXFP4_H"])
def test_tiny_linear_fwd_bwd(preset):
    """The tiny linear workload: X [512x256], W [256x256], dY [512x256]."""
    wl = inputs.workload("tiny")
    X, W, dY = wl["X"], wl["W"], wl["dY"]
    rec = Q.recipe(preset)
    seed = Q.make_seed(ROT, SRS)
    Y = Q.linear_fwd(X.cuda(), W.cuda(), rec, seed)
    dX, dW = Q.linear_bwd(dY.cuda(), X.cuda(), W.cuda(), rec, seed)
    Q.status()
    r = O.preset(preset)
    y_ref, y_b = O.linear_fwd(X, W, r, ROT, SRS)
    (dx_ref, dx_b), (dw_ref, dw_b) = O.linear_bwd(dY, X, W, r, ROT, SRS)
    within(Y, y_ref, y_b, True)
    within(dX, dx_ref, dx_b, True)
    within(dW, dw_ref, dw_b, False)


def test_tiny_linear_mxfp4_round_up():
    """The AMD MXFP4 recipe with the round-up shared exponent on all six
    operands (the tiny linear workload)."""
    import dataclasses
    wl = inputs.workload("tiny")
    X, W, dY = wl["X"], wl["W"], wl["dY"]
    rec = Q.recipe("AMD_MXFP4_H")
    for c in (rec.fprop, rec.dgrad, rec.wgrad):
        c.fmt = Q.MXFP4_RU
    seed = Q.make_seed(ROT, SRS)
    Y = Q.linear_fwd(X.cuda(), W.cuda(), rec, seed)
    dX, dW = Q.linear_bwd(dY.cuda(), X.cuda(), W.cuda(), rec, seed)
    Q.status()
    r0 = O.preset("AMD_MXFP4_H")
    r = O.Recipe(*(dataclasses.replace(c, fmt=O.MXFP4_RU) for c in (r0.fprop, r0.dgrad, r0.wgrad)))
    y_ref, y_b = O.linear_fwd(X, W, r, ROT, SRS)
    (dx_ref, dx_b), (dw_ref, dw_b) = O.linear_bwd(dY, X, W, r, ROT, SRS)
    within(Y, y_ref, y_b, True)
    within(dX, dx_ref, dx_b, True)
    within(dW, dw_ref, dw_b, False)


@pytest.mark.parametrize("hads", [(Q.HAD_NONE, Q.HAD_RAND16), (Q.HAD_RAND16, Q.HAD_RAND16)],
                         ids=["none-rand16", "rand16-rand16"])
def test_tiny_linear_nvfp4_rtn_backward(hads):
    """NVFP4 round-to-nearest on both backward GEMMs: dY's two quantizations
    come from one read (qfp4_quantize_dual), its tensor amaxes from two passes
    (different Hadamards) or one (the same)."""
    import dataclasses
    wl = inputs.workload("tiny")
    X, W, dY = wl["X"], wl["W"], wl["dY"]
    rec = Q.recipe("QUARTET2_NVFP4")
    for c, had in ((rec.dgrad, hads[0]), (rec.wgrad, hads[1])):
        c.rnd_a, c.rnd_b, c.had = Q.RTN, Q.RTN, had
    seed = Q.make_seed(ROT, SRS)
    dX, dW = Q.linear_bwd(dY.cuda(), X.cuda(), W.cuda(), rec, seed)
    Q.status()
    r0 = O.preset("QUARTET2_NVFP4")
    r = O.Recipe(r0.fprop, dataclasses.replace(r0.dgrad, rnd_a=O.RTN, rnd_b=O.RTN, had=hads[0]),
                 dataclasses.replace(r0.wgrad, rnd_a=O.RTN, rnd_b=O.RTN, had=hads[1]))
    (dx_ref, dx_b), (dw_ref, dw_b) = O.linear_bwd(dY, X, W, r, ROT, SRS)
    within(dX, dx_ref, dx_b, True)
    within(dW, dw_ref, dw_b, False)


def test_tiny_linear_dw_accumulate():
    """dw_accumulate = 1: dW += dY^T X into the caller's fp32 buffer (a main
    gradient across micro-batches); dX as without it."""
    wl = inputs.workload("tiny")
    X, W, dY = wl["X"], wl["W"], wl["dY"]
    rec = Q.recipe("QUARTET2_NVFP4")
    rec.dw_accumulate = 1
    seed = Q.make_seed(ROT, SRS)
    dW0 = inputs.normal(tuple(W.shape), 1.0, 3, "main_grad").float()
    dW = dW0.cuda()
    dX, dW = Q.linear_bwd(dY.cuda(), X.cuda(), W.cuda(), rec, seed, dW=dW)
    Q.status()
    r = O.preset("QUARTET2_NVFP4")
    (dx_ref, dx_b), (dw_ref, dw_b) = O.linear_bwd(dY, X, W, r, ROT, SRS)
    within(dX, dx_ref, dx_b, True)
    d0 = dW0.numpy().astype(np.float64)
    within(dW, d0 + dw_ref, dw_b + 2.0 ** -23 * (np.abs(d0) + np.abs(dw_ref)), False)


def test_autograd_function():
    wl = inputs.workload("tiny")
    X = wl["X"].cuda().requires_grad_(True)
    W = wl["W"].cuda().requires_grad_(True)
    rec = Q.recipe("QUARTET2_NVFP4")
    seed = Q.make_seed(ROT, SRS)
    Y = Q.Fp4Linear.apply(X, W, rec, seed)
    Y.backward(wl["dY"].cuda())
    Q.status()
    r = O.preset("QUARTET2_NVFP4")
    (dx_ref, dx_b), (dw_ref, dw_b) = O.linear_bwd(wl["dY"], wl["X"], wl["W"], r, ROT, SRS)
    within(X.grad, dx_ref, dx_b, True)
    within(W.grad, dw_ref, dw_b, True)


def test_linear_estimates_bf16_product():
    """Sanity (not parity): the FP4 layer's outputs track the bf16 products."""
    wl = inputs.workload("tiny")
    X, W, dY = (wl[k].cuda() for k in ("X", "W", "dY"))
    rec = Q.recipe("QUARTET2_NVFP4")
    seed = Q.make_seed(ROT, SRS)
    Y = Q.linear_fwd(X, W, rec, seed).float()
    dX, dW = Q.linear_bwd(dY, X, W, rec, seed)
    for got, ref in ((Y, X.float() @ W.float().T), (dX.float(), dY.float() @ W.float()),
                     (dW.float(), dY.float().T @ X.float())):
        rel = (got - ref).norm() / ref.norm()
        assert rel < 0.2, rel


def test_linear_rejects_bad_shapes():
    X = torch.zeros((100, 256), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((256, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(Q.QFP4Error):
        Q.linear_fwd(X, W, Q.recipe("NVIDIA_NVFP4"), Q.make_seed())


def test_calls_from_a_worker_thread():
    """A thread that never set a device (as a framework's worker thread may be)
    still runs the library on the caller's stream's context."""
    import threading
    wl = inputs.workload("tiny")
    X, W, dY = (wl[k].cuda() for k in ("X", "W", "dY"))
    rec = Q.recipe("QUARTET2_NVFP4")
    seed = Q.make_seed(ROT, SRS)
    ref_dX, ref_dW = Q.linear_bwd(dY, X, W, rec, seed)
    torch.cuda.synchronize()
    out = {}

    def worker():
        try:
            s = torch.cuda.Stream(device=X.device)
            out["dX"], out["dW"] = Q.linear_bwd(dY, X, W, rec, seed, stream=s)
            s.synchronize()
            out["dX0"], out["dW0"] = Q.linear_bwd(dY, X, W, rec, seed)  # default stream
            torch.cuda.synchronize()
        except Exception as e:  # noqa: BLE001
            out["err"] = e

    t = threading.Thread(target=worker)
    t.start()
    t.join()
    assert "err" not in out, out.get("err")
    for k in ("dX", "dX0"):
        assert torch.equal(out[k], ref_dX)
    for k in ("dW", "dW0"):
        assert torch.equal(out[k], ref_dW)


@pytest.mark.parametrize("M", [512, 128], ids=["pair", "single"])
@pytest.mark.parametrize("had", [Q.HAD_NONE, Q.HAD_DET16, Q.HAD_RAND16], ids=["none", "det16", "rand16"])
def test_linear_fwd_chain(had, M):
    """Two stacked layers through qfp4_linear_fwd_chain: layer 1's output Y1
    comes with its NVFP4 tensor amax for layer 2's Fprop rotation (from the
    GEMM epilogue with the CTA-pair kernel, M = 512; by an amax pass with the
    single-CTA one, M = 128), and layer 2 takes it for its input. Both outputs
    equal qfp4_linear_fwd's bit for bit, and the amax equals qfp4_amax of Y1
    with layer 2's sign vector (its seed's rot key, stream 0)."""
    K, N1, N2 = 256, 384, 256
    X = inputs.normal_with_outliers((M, K), 51, "cx").cuda()
    W1 = inputs.normal((N1, K), 0.05, 51, "cw1").cuda()
    W2 = inputs.normal((N2, N1), 0.05, 51, "cw2").cuda()
    rec = Q.recipe("QUARTET2_NVFP4")
    rec.fprop.had = had
    s1, s2 = Q.make_seed(11, 12), Q.make_seed(21, 22)
    Y1, a1 = Q.linear_fwd_chain(X, W1, rec, s1, next_had=had, next_seed=s2)
    Y2, none = Q.linear_fwd_chain(Y1, W2, rec, s2, x_amax=a1, want_y_amax=False)
    R1 = Q.linear_fwd(X, W1, rec, s1)
    R2 = Q.linear_fwd(Y1, W2, rec, s2)
    ref = Q.amax(Y1, had, Q.ROW, Q.make_seed(21, 0, 0, 0))
    torch.cuda.synchronize()
    Q.status()
    assert none is None
    assert torch.equal(Y1, R1) and torch.equal(Y2, R2)
    assert float(a1.cpu()[0]) == float(ref.cpu()[0]) > 0.0


@pytest.mark.parametrize("preset", ["QUARTET2_NVFP4", "NVIDIA_NVFP4"])
def test_plain_launches_give_the_same_results(preset, monkeypatch):
    """Programmatic dependent launch (the default) only changes when each
    kernel's set-up runs: with QFP4_PDL=0 (plain launches) a linear fwd+bwd on
    a layer of a few dozen launches, back to back on one stream, gives
    byte-identical outputs."""
    g = torch.Generator(device="cpu").manual_seed(3)
    X = (torch.randn((1024, 768), generator=g)).to(torch.bfloat16).cuda()
    W = (torch.randn((640, 768), generator=g) * 0.02).to(torch.bfloat16).cuda()
    dY = (torch.randn((1024, 640), generator=g) * 1e-3).to(torch.bfloat16).cuda()
    rec = Q.recipe(preset)
    seed = Q.make_seed(ROT, SRS)
    outs = {}
    for pdl in ("1", "0"):
        monkeypatch.setenv("QFP4_PDL", pdl)
        res = []
        for _ in range(3):
            res.append(Q.linear_fwd(X, W, rec, seed))
            res.extend(Q.linear_bwd(dY, X, W, rec, seed))
        torch.cuda.synchronize()
        Q.status()
        outs[pdl] = res
    for a, b in zip(outs["1"], outs["0"]):
        assert torch.equal(a, b)
