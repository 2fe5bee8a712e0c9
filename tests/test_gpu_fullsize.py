"""The benchmark's layers at their full sizes (the MLP up/gate layer, the
attention QKV projection, the MLP down layer at 2048, 16384 and 32768 tokens),
in the launch configuration bench.py times: the six quantizations of one linear fwd+bwd (with the fused
row-and-column amax of dY, and its row and column quantizations from one read,
where the recipe allows them) and the three GEMMs.

Checked on samples the oracle computes one by one: 64 rows of every quantized
operand (first and last rows, the rows around a 128-row tile edge, random
rows) bit for bit, codes, scales and tensor scale; and for every GEMM the
64 x 64 outputs of 64 sampled rows of A and of B against fp64 dot products of
the oracle's own quantization of those rows, within 2^-18 * sum |a b| (bf16
outputs add 2^-8 |D|). The oracle quantizes only the sampled rows, with the
tensor amax and the random words of the whole tensor."""
import numpy as np
import pytest
import torch

import oracle as O
from fp4_precision_b200 import inputs
from fp4_precision_b200 import qfp4 as Q

import helpers

pytestmark = pytest.mark.gpu

ROT, SR = 0x0123_4567, 0x89AB_CDEF
LAYERS = [("mlp_up", "QUARTET2_NVFP4", None), ("mlp_up", "AMD_MXFP4_H", None), ("mlp_down", "NVIDIA_NVFP4", 16384),
          ("qkv", "QUARTET2_NVFP4", None), ("mlp_down", "QUARTET2_NVFP4", 2048), ("mlp_down", "NVIDIA_NVFP4", 32768),
          ("mlp_down", "QUARTET2_NVFP4", 32768)]


def sample_rows(n, rng, count=64):
    fixed = [0, 1, 127, 128, 255, 256, n - 129, n - 128, n - 2, n - 1]
    rest = rng.choice(n, size=count - len(fixed), replace=False)
    return np.unique(np.clip(np.concatenate([fixed, rest]), 0, n - 1))


def oracle_rows(t_cpu, fmt, rnd, had, axis, g, o, rows):
    return O.quantize(t_cpu, fmt, rnd, had, axis, ROT, g, SR, o, rows_sel=rows)


def assert_rows_same(q_gpu, q_ref, rows, fmt):
    nb = O.BLOCK[fmt]
    codes = q_gpu.codes.index_select(0, torch.as_tensor(rows, device=q_gpu.codes.device)).cpu().numpy()
    assert np.array_equal(codes, q_ref.codes), f"{np.sum(codes != q_ref.codes)} code bytes differ"
    flat = helpers.to_numpy_u8(q_gpu.scales)
    kb = q_gpu.k // nb
    sc = flat[helpers.atom_offset(q_gpu.rows, kb, np.asarray(rows)[:, None], np.arange(kb)[None, :])]
    assert np.array_equal(sc, q_ref.scales), f"{np.sum(sc != q_ref.scales)} scales differ"
    g = float(q_gpu.tensor_scale.cpu()[0])
    assert np.float32(g).tobytes() == np.float32(q_ref.g).tobytes(), (g, q_ref.g)


@pytest.mark.parametrize("workload,preset,M", LAYERS, ids=[f"{w}-{p}" + (f"-M{m}" if m else "") for w, p, m in LAYERS])
def test_layer_full_size_sampled(workload, preset, M):
    dev = torch.device("cuda", 0)
    wl = inputs.workload(workload, device=dev, M=M)
    X, W, dY = wl["X"], wl["W"], wl["dY"]
    rec = Q.recipe(preset)
    c = rec.fprop, rec.dgrad, rec.wgrad
    # (tensor, cfg, rounding, axis, gemm g, operand o): as the bench's step and qfp4_linear_*
    ops = [(X, c[0], c[0].rnd_a, Q.ROW, 0, 0), (W, c[0], c[0].rnd_b, Q.ROW, 0, 1),
           (dY, c[1], c[1].rnd_a, Q.ROW, 1, 2), (W, c[1], c[1].rnd_b, Q.COL, 1, 3),
           (dY, c[2], c[2].rnd_a, Q.COL, 2, 4), (X, c[2], c[2].rnd_b, Q.COL, 2, 5)]
    ws = torch.empty((Q.quantize_workspace_bytes(),), dtype=torch.uint8, device=dev)
    # dY as the layer quantizes it: both tensor amaxes from one pass (NVFP4, same
    # Hadamard), both quantizations from one read (round-to-nearest)
    had_n = {Q.HAD_NONE: 0, Q.HAD_DET16: 16, Q.HAD_DET32: 32, Q.HAD_RAND16: 16, Q.HAD_RAND32: 32}
    fused = (c[1].fmt == Q.NVFP4 and c[2].fmt == Q.NVFP4 and c[1].had == c[2].had
             and c[1].had in (Q.HAD_NONE, Q.HAD_DET16, Q.HAD_RAND16))
    dual = (c[1].fmt == c[2].fmt and c[1].rnd_a == Q.RTN and c[2].rnd_a == Q.RTN
            and had_n[c[1].had] in (0, had_n[c[2].had]))
    s_row, s_col = Q.make_seed(ROT, SR, 1, 2), Q.make_seed(ROT, SR, 2, 4)
    dy_amax = torch.empty((2,), dtype=torch.float32, device=dev)
    if fused:
        Q.amax_rowcol(dY, c[1].had, s_row, s_col, out=dy_amax, workspace=ws)
    elif dual and c[1].fmt == Q.NVFP4:
        Q.amax(dY, c[1].had, Q.ROW, s_row, out=dy_amax[0:1], workspace=ws)
        Q.amax(dY, c[2].had, Q.COL, s_col, out=dy_amax[1:2], workspace=ws)
    qs = [None] * 6
    if dual:
        nv = c[1].fmt == Q.NVFP4
        qs[2], qs[4] = Q.quantize_dual(dY, c[1].fmt, Q.RTN, c[1].had, c[2].had, s_row, s_col,
                                       dy_amax[0:1] if nv else None, dy_amax[1:2] if nv else None)
    for i, (t, cfg, rnd, axis, g, o) in enumerate(ops):
        if qs[i] is not None:
            continue
        am = None
        if fused and i in (2, 4):
            am = dy_amax[0:1] if i == 2 else dy_amax[1:2]
        qs[i] = Q.quantize(t, cfg.fmt, rnd, cfg.had, axis, Q.make_seed(ROT, SR, g, o), amax_in=am, workspace=ws)
    Y = Q.gemm(qs[0], qs[1], torch.bfloat16)
    dX = Q.gemm(qs[2], qs[3], torch.bfloat16)
    dW = Q.gemm(qs[4], qs[5], torch.float32)
    torch.cuda.synchronize()
    Q.status()

    rng = np.random.default_rng(7)
    cpu = {"X": X.cpu(), "W": W.cpu(), "dY": dY.cpu()}
    names = ["X", "W", "dY", "W", "dY", "X"]
    picked = [sample_rows(q.rows, rng) for q in qs]
    refs = []
    for i, (t, cfg, rnd, axis, g, o) in enumerate(ops):
        ref = oracle_rows(cpu[names[i]], cfg.fmt, rnd, cfg.had, axis, g, o, picked[i])
        assert_rows_same(qs[i], ref, picked[i], cfg.fmt)
        refs.append(ref)
    for a, b, D, bf16 in ((0, 1, Y, True), (2, 3, dX, True), (4, 5, dW, False)):
        Ad, Bd = O.dequantize(refs[a]), O.dequantize(refs[b])
        ref = Ad @ Bd.T
        bound = O.GEMM_REL_BOUND * (np.abs(Ad) @ np.abs(Bd).T)
        ri = torch.as_tensor(picked[a], device=D.device)
        ci = torch.as_tensor(picked[b], device=D.device)
        got = D.index_select(0, ri).index_select(1, ci).float().cpu().numpy().astype(np.float64)
        tol = bound + (2.0 ** -8 * np.abs(ref) if bf16 else 0.0)
        err = np.abs(got - ref)
        assert np.all(err <= tol), f"GEMM {a // 2}: {np.sum(err > tol)} of {err.size} sampled outputs out of bound"
