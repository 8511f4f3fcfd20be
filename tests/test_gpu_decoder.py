"""GPU parity on the 32-layer Llama-7B-shaped decoder workload: every linear
of every layer (q, k, v, o 4096 x 4096; gate, up 11008 x 4096; down
4096 x 11008; 224 weights, 6.5e9 parameters) is quantised and dequantised on
the GPU through the C-ABI and checked bit-exact against the oracle in full
(every packed byte, FP8 scale code, meta scale and dequantised bf16, compared
as SHA-256 digests of the whole byte streams, the oracle running in a pool of
spawned processes); a sample of layers runs forward and backward at 4096
tokens and is checked against the oracle's fp64 products on 256 sampled token
rows of Y and dX and on the whole of T, dA and dB."""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

from oracle import nf4_oracle as o
from bit_nf4_quantised_b200 import synthetic as syn

from _parity import assert_close, oracle_wtilde

pytestmark = pytest.mark.gpu

WORKLOAD = "llama7b_decoder_32layers_m4096_r16"
# (layer, linear) pairs run through the full forward and backward: every
# linear of the first layer and three shapes of the last
SAMPLED_LAYERS = ((0, None), (31, ("o", "up", "down")))


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import bit_nf4_quantised_b200 as pkg
    pkg.lib()
    return pkg


def test_decoder_weights_all_224_in_full(q):
    """All 224 weights quantised and dequantised on the GPU and compared with
    the oracle's in full."""
    import _oracle_pool as op
    lins = syn.WORKLOADS[WORKLOAD].layers
    assert len(lins) == 224
    with op.pool() as px:
        want = [px.submit(op.oracle_storage_digests, lin) for lin in lins]
        # the seeded weights are generated on host threads a few ahead (numpy's
        # generator releases the GIL), bounding the host memory held at once
        workers = max(1, min(6, os.cpu_count() or 1))
        ex = ThreadPoolExecutor(workers)
        make = lambda lin: syn.make_weight(lin, np.random.default_rng(lin.seed))
        pending = [ex.submit(make, lin) for lin in lins[:workers]]
        got = []
        for i, lin in enumerate(lins):
            W = pending.pop(0).result()
            if i + workers < len(lins):
                pending.append(ex.submit(make, lins[i + workers]))
            w = q.qlora_quantize(torch.from_numpy(W).cuda())
            deq = q.qlora_dequantize(w)
            got.append(op.gpu_storage_digests(w, deq))
            del w, deq, W
        ex.shutdown()
        for lin, g, f in zip(lins, got, want):
            assert g == f.result(), f"{lin.name}: stored bytes or W~ differ from the oracle"


def _sampled_linears():
    lins = syn.WORKLOADS[WORKLOAD].layers
    out = []
    for layer, names in SAMPLED_LAYERS:
        for lin in lins:
            lname, nm = lin.name.split(".")
            if lname == f"layer{layer}" and (names is None or nm in names):
                out.append(lin)
    return out


@pytest.mark.parametrize("lin", _sampled_linears(), ids=lambda l: l.name)
def test_decoder_layer_forward_backward(q, lin):
    d = syn.make_layer(lin)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    w = q.qlora_quantize(torch.from_numpy(d["W"]).cuda())
    ws = q.workspace(lin.M, lin.N, lin.K, lin.r)
    T = torch.empty(lin.M, lin.r, dtype=torch.float32, device="cuda")
    Y = q.qlora_linear_forward(g["X"], w, g["A"], g["B"], lin.gamma, T_save=T, ws=ws)
    dX, dA, dB = q.qlora_linear_backward(g["dY"], g["X"], w, g["A"], g["B"], lin.gamma,
                                         T_saved=T, ws=ws)
    torch.cuda.synchronize()
    assert q.device_error_word(ws) == 0
    Wt = oracle_wtilde(o.quantize(d["W"]), lin.N, lin.K)
    X, A, B, dY = (syn.as_f64(d[k]) for k in ("X", "A", "B", "dY"))
    rows = np.unique(np.concatenate([[0, 511, 512, lin.M - 1],
                                     np.random.default_rng(lin.seed).integers(0, lin.M, 252)]))
    r_t = torch.from_numpy(rows).cuda()
    Xs, dYs = X[rows], dY[rows]
    assert_close(f"{lin.name} Y rows", Y[r_t], Xs @ Wt.T + lin.gamma * (Xs @ A.T) @ B.T)
    assert_close(f"{lin.name} dX rows", dX[r_t], dYs @ Wt + lin.gamma * (dYs @ B) @ A)
    Tr = X @ A.T
    assert_close(f"{lin.name} T", T, Tr)
    assert_close(f"{lin.name} dA", dA, lin.gamma * (dY @ B).T @ X)
    assert_close(f"{lin.name} dB", dB, lin.gamma * dY.T @ Tr)
