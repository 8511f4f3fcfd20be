"""GPU parity of layer chaining with gradient checkpointing (the SwiGLU MLP
of adapted NF4 linears, qlora_mlp_forward / qlora_mlp_backward) against the
oracle's mlp_forward / mlp_backward in fp64 on the oracle's own W~, with the
activations between the steps in bf16 (the pages' compute type): Y and dX
in full, and dA, dB of all six adapter matrices, within a relative Frobenius
error of 1e-2 and a per-element error of 5e-2 * rms.  The Llama-7B MLP
workload (8192 tokens, D = 4096, F = 11008, r = 64, alpha = 16) runs in
full; the oracle takes it in chunks of tokens (its gradients summed), which
is exact because every token's forward and backward is independent and the
adapter gradients are sums over tokens."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import nf4_oracle as o
from bit_nf4_quantised_b200 import synthetic as syn

from _parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import bit_nf4_quantised_b200 as pkg
    pkg.lib()
    return pkg


def _make(q, lins, M):
    """Stored weights and adapters of gate, up, down (one seeded layer each);
    X from the gate layer's draw, dY from the down layer's."""
    host = {}
    dev = {}
    for lin, name in zip(lins, ("gate", "up", "down")):
        d = syn.make_layer(syn.Linear(lin.name, M, lin.N, lin.K, lin.r, lin.alpha, lin.sigma,
                                      lin.outliers, lin.seed))
        host[name] = d
        dev[name] = q.qlora_quantize(torch.from_numpy(d["W"]).cuda())
    mlp = q.MLP(dev["gate"], dev["up"], dev["down"],
                host["gate"]["A"].cuda(), host["gate"]["B"].cuda(),
                host["up"]["A"].cuda(), host["up"]["B"].cuda(),
                host["down"]["A"].cuda(), host["down"]["B"].cuda())
    X = host["gate"]["X"]
    dY = host["down"]["dY"]
    return host, mlp, X, dY


def _oracle(host, X, dY, gamma, chunk=1024):
    layers = {}
    for name in ("gate", "up", "down"):
        d = host[name]
        W = d["W"]
        Wt = o.dequantize(*o.quantize(W), W.shape[0], W.shape[1]).astype(np.float64)
        layers[name] = (Wt, syn.as_f64(d["A"]), syn.as_f64(d["B"]))
    X64, dY64 = syn.as_f64(X), syn.as_f64(dY)
    M = X64.shape[0]
    Y = np.empty_like(X64)
    dX = np.empty_like(X64)
    grads = None
    for m0 in range(0, M, chunk):
        xs, ds = X64[m0:m0 + chunk], dY64[m0:m0 + chunk]
        Y[m0:m0 + chunk], saved = o.mlp_forward(xs, layers, gamma, bf16_activations=True)
        dx, g = o.mlp_backward(ds, xs, layers, gamma, saved, bf16_activations=True)
        dX[m0:m0 + chunk] = dx
        if grads is None:
            grads = {k: [v[0].copy(), v[1].copy()] for k, v in g.items()}
        else:
            for k, v in g.items():
                grads[k][0] += v[0]
                grads[k][1] += v[1]
    return Y, dX, grads


def _check(q, lins, M, gamma, accumulate=False):
    host, mlp, X, dY = _make(q, lins, M)
    ws = q.mlp_workspace(M, mlp)
    Y = q.qlora_mlp_forward(X.cuda(), mlp, gamma, ws=ws)
    torch.cuda.synchronize()
    assert q.device_error_word(ws) == 0
    g0 = None
    if accumulate:
        g0 = {}
        for lin, name in ((mlp.gate, "gate"), (mlp.up, "up"), (mlp.down, "down")):
            g0[f"dA_{name}"] = torch.full((mlp.r, lin.cols), 0.5, dtype=torch.float32, device="cuda")
            g0[f"dB_{name}"] = torch.full((lin.rows, mlp.r), -0.25, dtype=torch.float32, device="cuda")
    base = {k: v.clone() for k, v in g0.items()} if g0 else None
    dX, grads = q.qlora_mlp_backward(dY.cuda(), X.cuda(), mlp, gamma, grads=g0,
                                     accumulate=accumulate, ws=ws)
    torch.cuda.synchronize()
    assert q.device_error_word(ws) == 0
    Yr, dXr, gr = _oracle(host, X, dY, gamma)
    assert_close("Y", Y, Yr)
    assert_close("dX", dX, dXr)
    for name in ("gate", "up", "down"):
        dA, dB = grads[f"dA_{name}"], grads[f"dB_{name}"]
        if base:
            dA, dB = dA - base[f"dA_{name}"], dB - base[f"dB_{name}"]
        assert_close(f"dA_{name}", dA, gr[name][0])
        assert_close(f"dB_{name}", dB, gr[name][1])


def _small(D, F, r, alpha, seed):
    return (syn.Linear("gate", 0, F, D, r, alpha, 0.02, True, seed),
            syn.Linear("up", 0, F, D, r, alpha, 0.02, True, seed + 1),
            syn.Linear("down", 0, D, F, r, alpha, 0.02, True, seed + 2))


@pytest.mark.parametrize("M,D,F,r", [(100, 256, 640, 8), (12, 512, 768, 16), (513, 320, 1088, 24)])
def test_mlp_small_ragged(q, M, D, F, r):
    lins = _small(D, F, r, 2.0 * r, seed=D + F)
    _check(q, lins, M, lins[0].gamma)


def test_mlp_accumulates_adapter_gradients(q):
    lins = _small(256, 512, 16, 32.0, seed=9)
    _check(q, lins, 64, lins[0].gamma, accumulate=True)


def test_mlp_llama7b_shapes(q):
    lins = syn.WORKLOADS["llama7b_mlp_m8192_r64"].layers
    _check(q, lins, lins[0].M, lins[0].gamma)


def test_mlp_empty_batch(q):
    lins = _small(256, 512, 8, 16.0, seed=3)
    host, mlp, X, dY = _make(q, lins, 4)
    grads = {}
    for lin, name in ((mlp.gate, "gate"), (mlp.up, "up"), (mlp.down, "down")):
        grads[f"dA_{name}"] = torch.ones(mlp.r, lin.cols, dtype=torch.float32, device="cuda")
        grads[f"dB_{name}"] = torch.ones(lin.rows, mlp.r, dtype=torch.float32, device="cuda")
    e = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    Y = q.qlora_mlp_forward(e, mlp, 2.0)
    dX, g = q.qlora_mlp_backward(e, e, mlp, 2.0, grads=grads)
    torch.cuda.synchronize()
    assert Y.shape == (0, 256) and dX.shape == (0, 256)
    assert all(float(v.abs().max()) == 0.0 for v in g.values())
