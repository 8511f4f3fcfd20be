"""GPU parity of the adapted linear layer through the C-ABI: Y, T, dX, dA and
dB of the tcgen05 dequant-GEMM path (M > 16) and the dequant-GEMV path
(M <= 16) against the oracle's fp64 products on the oracle's own W~, within
a relative Frobenius error of 1e-2 and a per-element error of 5e-2 * rms."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import nf4_oracle as o
from bit_nf4_quantised_b200 import synthetic as syn

from _parity import assert_close, groups_of_rows, oracle_wtilde

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import bit_nf4_quantised_b200 as pkg
    pkg.lib()
    return pkg


def _gpu_inputs(d):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def _run(q, lin, with_T=True, accumulate=False, want_dX=True):
    d = syn.make_layer(lin)
    g = _gpu_inputs(d)
    w = q.qlora_quantize(torch.from_numpy(d["W"]).cuda())
    ws = q.workspace(lin.M, lin.N, lin.K, lin.r)
    T = torch.empty(lin.M, lin.r, dtype=torch.float32, device="cuda")
    Y = q.qlora_linear_forward(g["X"], w, g["A"], g["B"], lin.gamma, T_save=T, ws=ws)
    torch.cuda.synchronize()
    assert q.device_error_word(ws) == 0
    dA0 = torch.ones(lin.r, lin.K, dtype=torch.float32, device="cuda") if accumulate else None
    dB0 = torch.ones(lin.N, lin.r, dtype=torch.float32, device="cuda") if accumulate else None
    dX, dA, dB = q.qlora_linear_backward(g["dY"], g["X"], w, g["A"], g["B"], lin.gamma,
                                         T_saved=T if with_T else None, dA=dA0, dB=dB0,
                                         accumulate=accumulate, want_dX=want_dX, ws=ws)
    torch.cuda.synchronize()
    assert q.device_error_word(ws) == 0
    return d, w, Y, T, dX, dA, dB


def _reference(d, lin):
    Wt = oracle_wtilde(o.quantize(d["W"]), lin.N, lin.K)
    X, A, B, dY = (syn.as_f64(d[k]) for k in ("X", "A", "B", "dY"))
    Y, T = o.linear_forward(X, Wt, A, B, lin.gamma)
    dX, dA, dB, _ = o.linear_backward(dY, X, Wt, A, B, lin.gamma)
    return Y, T, dX, dA, dB


CASES = [
    # (M, N, K, r)           GEMM path (M > 16)
    (64, 256, 512, 8),       # the single-layer config
    (200, 264, 320, 16),     # ragged M, N and K tiles
    (300, 520, 192, 24),     # rank not a multiple of 16
    (129, 256, 256, 64),
    (256, 512, 1024, 128),   # two LoRA tail steps
    (17, 136, 128, 8),       # one token above the GEMV threshold
    (4608, 2200, 2304, 16),  # two waves: per-pair column runs (forward 288, dX 384 wide)
    #                         GEMV path (M <= 16)
    (1, 1000, 2048, 16),
    (4, 512, 4160, 16),      # ragged last contraction slice
    (16, 776, 1024, 32),
    (8, 264, 192, 8),
    (9, 256, 4096, 64),
    (16, 1024, 2048, 128),
    (4, 512, 4352, 16),      # 17 contraction chunks of 256: many one-chunk slices
    (2, 4104, 2304, 8),      # ragged last row tile, half-filled last weight tile
    (12, 40, 768, 24),
]


@pytest.mark.parametrize("M,N,K,r", CASES)
def test_forward_backward(q, M, N, K, r):
    lin = syn.Linear("case", M, N, K, r, alpha=2.0 * r, outliers=True, seed=M * 7 + N + K + r)
    d, w, Y, T, dX, dA, dB = _run(q, lin)
    Yr, Tr, dXr, dAr, dBr = _reference(d, lin)
    assert_close("Y", Y, Yr)
    assert_close("T", T, Tr)
    assert_close("dX", dX, dXr)
    assert_close("dA", dA, dAr)
    assert_close("dB", dB, dBr)


@pytest.mark.parametrize("M,N,K,r", [(1, 1000, 2048, 16), (4, 512, 4352, 16), (16, 1024, 2048, 128),
                                     (9, 256, 4096, 64), (200, 264, 320, 16), (4608, 2200, 2304, 16)])
def test_same_inputs_same_bytes(q, M, N, K, r):
    """Every result is reproducible: three forward + backward calls on the
    same inputs give the same bytes of Y, T, dX, dA and dB (no reduction
    depends on the order in which warps or CTAs finish)."""
    lin = syn.Linear("case", M, N, K, r, alpha=2.0 * r, outliers=True, seed=M + N + K + r)
    d = syn.make_layer(lin)
    g = _gpu_inputs(d)
    w = q.qlora_quantize(torch.from_numpy(d["W"]).cuda())
    outs = []
    for _ in range(3):
        T = torch.empty(M, r, dtype=torch.float32, device="cuda")
        Y = q.qlora_linear_forward(g["X"], w, g["A"], g["B"], lin.gamma, T_save=T)
        dX, dA, dB = q.qlora_linear_backward(g["dY"], g["X"], w, g["A"], g["B"], lin.gamma,
                                             T_saved=T)
        torch.cuda.synchronize()
        outs.append([t.view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32).cpu()
                     for t in (Y, T, dX, dA, dB)])
    for other in outs[1:]:
        for name, a, b in zip(("Y", "T", "dX", "dA", "dB"), outs[0], other):
            assert torch.equal(a, b), name


def test_decode_same_bytes_full_size(q):
    """The decode GEMV with 16 tokens over 8192 x 28672 (many CTAs share T):
    the same Y bytes on every call."""
    lin = syn.WORKLOADS["decode_gemv_8192x28672_m16"].layers[0]
    d = syn.make_layer(lin, with_grad=False)
    g = _gpu_inputs(d)
    w = q.qlora_quantize(torch.from_numpy(d["W"]).cuda())
    Ys = [q.qlora_linear_forward(g["X"], w, g["A"], g["B"], lin.gamma).view(torch.int16).cpu()
          for _ in range(4)]
    assert all(torch.equal(Ys[0], y) for y in Ys[1:])


def test_recompute_T_accumulate_and_no_dX(q):
    lin = syn.Linear("case", 96, 264, 384, 16, alpha=32.0, seed=3)
    d, w, Y, T, dX, dA, dB = _run(q, lin, with_T=False, accumulate=True, want_dX=False)
    _, _, _, dAr, dBr = _reference(d, lin)
    assert dX is None
    assert_close("dA+1", dA, dAr + 1.0)
    assert_close("dB+1", dB, dBr + 1.0)


def test_empty_batch(q):
    lin = syn.Linear("case", 0, 256, 512, 8, alpha=16.0)
    w = q.qlora_quantize(torch.randn(256, 512, device="cuda"))
    X = torch.empty(0, 512, dtype=torch.bfloat16, device="cuda")
    A = torch.randn(8, 512, device="cuda").bfloat16()
    B = torch.randn(256, 8, device="cuda").bfloat16()
    Y = q.qlora_linear_forward(X, w, A, B, 2.0)
    assert Y.shape == (0, 256)
    dY = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    dX, dA, dB = q.qlora_linear_backward(dY, X, w, A, B, 2.0)
    torch.cuda.synchronize()
    assert dX.shape == (0, 512) and float(dA.abs().max()) == 0 and float(dB.abs().max()) == 0


def test_attn_projection_full_size(q):
    """4096 tokens x 4096 x 4096, r = 16: Y and dX on 256 sampled token rows,
    dA and dB in full."""
    lin = syn.WORKLOADS["llama7b_attn_proj_4096x4096_m4096_r16"].layers[0]
    d, w, Y, T, dX, dA, dB = _run(q, lin)
    Wt = oracle_wtilde(o.quantize(d["W"]), lin.N, lin.K)
    X, A, B, dY = (syn.as_f64(d[k]) for k in ("X", "A", "B", "dY"))
    rows = np.unique(np.concatenate([[0, 127, 128, lin.M - 1],
                                     np.random.default_rng(1).integers(0, lin.M, 252)]))
    Xs, dYs = X[rows], dY[rows]
    Yr = Xs @ Wt.T + lin.gamma * (Xs @ A.T) @ B.T
    dXr = dYs @ Wt + lin.gamma * (dYs @ B) @ A
    assert_close("Y rows", Y[torch.from_numpy(rows).cuda()], Yr)
    assert_close("dX rows", dX[torch.from_numpy(rows).cuda()], dXr)
    assert_close("T", T, X @ A.T)
    U = dY @ B
    assert_close("dA", dA, lin.gamma * U.T @ X)
    assert_close("dB", dB, lin.gamma * dY.T @ (X @ A.T))


@pytest.mark.parametrize("name", [f"decode_gemv_{nk}_m{m}" for nk in ("28672x8192", "8192x28672")
                                  for m in (1, 4, 16)])
def test_decode_full_size_sampled_columns(q, name):
    lin = syn.WORKLOADS[name].layers[0]
    d = syn.make_layer(lin, with_grad=False)
    g = _gpu_inputs(d)
    w = q.qlora_quantize(torch.from_numpy(d["W"]).cuda())
    Y = q.qlora_linear_forward(g["X"], w, g["A"], g["B"], lin.gamma)
    torch.cuda.synchronize()
    X, A, B = (syn.as_f64(d[k]) for k in ("X", "A", "B"))
    rng = np.random.default_rng(2)
    cols = np.unique(np.concatenate([[0, lin.N - 1], rng.integers(0, lin.N, 30)]))
    flat = d["W"].reshape(-1)
    ref = np.empty((lin.M, cols.size))
    for j, (n, (e0, e1)) in enumerate(zip(cols, groups_of_rows(cols, lin.K))):
        packed, sc, meta = o.quantize(flat[e0:e1])
        sub = o.bf16_bits_to_float(o.dequantize_bits(packed, sc, meta, e1 - e0)).astype(np.float64)
        wrow = sub[n * lin.K - e0:(n + 1) * lin.K - e0]
        ref[:, j] = X @ wrow + lin.gamma * (X @ A.T) @ B[n]
    assert_close(f"{name} Y cols", Y[:, torch.from_numpy(cols).cuda()], ref)


def test_mlp_full_size_sampled_rows(q):
    """gate (11008 x 4096) and down (4096 x 11008) at 8192 tokens, r = 64."""
    for lin in (syn.WORKLOADS["llama7b_mlp_m8192_r64"].layers[0],
                syn.WORKLOADS["llama7b_mlp_m8192_r64"].layers[2]):
        d, w, Y, T, dX, dA, dB = _run(q, lin)
        Wt = oracle_wtilde(o.quantize(d["W"]), lin.N, lin.K)
        X, A, B, dY = (syn.as_f64(d[k]) for k in ("X", "A", "B", "dY"))
        rows = np.unique(np.concatenate([[0, lin.M - 1],
                                         np.random.default_rng(4).integers(0, lin.M, 126)]))
        Xs, dYs = X[rows], dY[rows]
        r_t = torch.from_numpy(rows).cuda()
        assert_close("Y rows", Y[r_t], Xs @ Wt.T + lin.gamma * (Xs @ A.T) @ B.T)
        assert_close("dX rows", dX[r_t], dYs @ Wt + lin.gamma * (dYs @ B) @ A)
        assert_close("dA", dA, lin.gamma * (dY @ B).T @ X)
        assert_close("dB", dB, lin.gamma * dY.T @ (X @ A.T))
