"""Failure detection of the tensor-core GEMM: with its wait limit set far
below what a pipeline barrier takes (qlora_set_gemm_wait_limit_us), waits run
out on purpose (under a limit this short every poll checks the clock, and the
MMA issuer's waits for each step's loaded and dequantised tiles last longer
than a microsecond, on the 64-token 256 x 512 layer as on the 4096-token
one); the call still returns QLORA_OK, the forward's and the backward's
workspace error word carries bit 0 (a bounded wait expired),
the kernel winds down on its own (in-flight copies and MMAs land, tensor
memory is freed), and the next call with the default limit on the same stream
computes the layer correctly.  No fault, trap or hang is involved: every wait
is bounded and the expiry is an ordinary status."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import nf4_oracle as o
from bit_nf4_quantised_b200 import synthetic as syn

from _parity import assert_close, oracle_wtilde

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import bit_nf4_quantised_b200 as pkg
    pkg.lib()
    yield pkg
    pkg.lib().qlora_set_gemm_wait_limit_us(0)


def test_wait_limit_arguments(q):
    L = q.lib()
    assert L.qlora_set_gemm_wait_limit_us(-1) == q._lib.QLORA_ERR_UNSUPPORTED
    assert L.qlora_set_gemm_wait_limit_us(20_000_000) == q._lib.QLORA_ERR_UNSUPPORTED
    assert L.qlora_set_gemm_wait_limit_us(0) == q._lib.QLORA_OK


@pytest.mark.parametrize("workload", ["single_256x512_m64_r8", "llama7b_attn_proj_4096x4096_m4096_r16"])
def test_expired_waits_are_reported_and_the_next_call_is_correct(q, workload):
    L = q.lib()
    lin = syn.WORKLOADS[workload].layers[0]
    d = syn.make_layer(lin)
    g = {k: d[k].cuda() for k in ("X", "A", "B", "dY")}
    w = q.qlora_quantize(torch.from_numpy(d["W"]).cuda())
    ws = q.workspace(lin.M, lin.N, lin.K, lin.r)
    expired_fwd = expired_bwd = 0
    try:
        assert L.qlora_set_gemm_wait_limit_us(1) == q._lib.QLORA_OK
        for _ in range(3):
            # each call clears its error word on entry: read it after each
            q.qlora_linear_forward(g["X"], w, g["A"], g["B"], lin.gamma, ws=ws)
            torch.cuda.synchronize()
            word = q.device_error_word(ws)
            assert word & ~1 == 0, f"unexpected error bits {word:#x}"
            expired_fwd += word & 1
            q.qlora_linear_backward(g["dY"], g["X"], w, g["A"], g["B"], lin.gamma, ws=ws)
            torch.cuda.synchronize()
            word = q.device_error_word(ws)
            assert word & ~1 == 0, f"unexpected error bits {word:#x}"
            expired_bwd += word & 1
    finally:
        assert L.qlora_set_gemm_wait_limit_us(0) == q._lib.QLORA_OK
    # every step is waited for by the MMA issuer while its weight tile is
    # loaded and dequantised: more than a microsecond per wait
    assert expired_fwd >= 1 and expired_bwd >= 1, \
        f"waits ran out in {expired_fwd} forward and {expired_bwd} backward calls of 3"
    T = torch.empty(lin.M, lin.r, dtype=torch.float32, device="cuda")
    Y = q.qlora_linear_forward(g["X"], w, g["A"], g["B"], lin.gamma, T_save=T, ws=ws)
    dX, dA, dB = q.qlora_linear_backward(g["dY"], g["X"], w, g["A"], g["B"], lin.gamma,
                                         T_saved=T, ws=ws)
    torch.cuda.synchronize()
    assert q.device_error_word(ws) == 0
    rows = np.unique(np.concatenate([[0, lin.M - 1],
                                     np.random.default_rng(1).integers(0, lin.M, 62)]))
    Wt = oracle_wtilde(o.quantize(d["W"]), lin.N, lin.K)
    X, A, B, dY = (syn.as_f64(d[k]) for k in ("X", "A", "B", "dY"))
    r_t = torch.from_numpy(rows).cuda()
    Xs, dYs = X[rows], dY[rows]
    assert_close("Y rows", Y[r_t], Xs @ Wt.T + lin.gamma * (Xs @ A.T) @ B.T)
    assert_close("dX rows", dX[r_t], dYs @ Wt + lin.gamma * (dYs @ B) @ A)
    assert_close("dA", dA, lin.gamma * (dY @ B).T @ X)
    assert_close("dB", dB, lin.gamma * dY.T @ (X @ A.T))
