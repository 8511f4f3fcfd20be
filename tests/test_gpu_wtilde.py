"""Both linear paths multiply the W~ of "The forward pass and gradients",
bf16_rne(fp32(q[idx] * c~)), and nothing else: the tcgen05 dequant-GEMM
(M > 16) and the dequant-GEMV (M <= 16) are checked against X W~^T built
from the oracle's W~, with the adapter's B set to zero so that only the
stored weight contributes.

  - One-hot activations: each output is then one weight of W~, with no
    accumulation at all, so Y must equal the oracle's W~ bit for bit.
  - Random activations: Y must lie within one bf16 rounding of the exact
    X W~^T widened by the fp32 accumulation bound (K + 16) 2^-24 sum|x w~|,
    and at least 99% of the outputs must equal bf16_rne(X W~^T) exactly.
    A path that rounded the code before scaling it (bf16(q) * c~) misses
    both by a wide margin."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import nf4_oracle as o
from bit_nf4_quantised_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import bit_nf4_quantised_b200 as pkg
    pkg.lib()
    return pkg


def _bits_to_f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _store(q, N, K, seed):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02))
    W.reshape(-1)[rng.choice(N * K, N * K // 1000, replace=False)] *= np.float32(10.0)
    w = q.qlora_quantize(torch.from_numpy(W).cuda())
    Wt = o.dequantize(*o.quantize(W), N, K).astype(np.float64)
    return w, Wt


def _forward(q, w, X, r, N, K):
    A = (torch.randn(r, K, device="cuda") / K ** 0.5).bfloat16()
    B = torch.zeros(N, r, dtype=torch.bfloat16, device="cuda")
    Y = q.qlora_linear_forward(X, w, A, B, 2.0)
    torch.cuda.synchronize()
    return Y.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("M", [1, 4, 16, 64])
def test_one_hot_rows_return_wtilde_exactly(q, M):
    N, K, r = 512, 2048, 16
    w, Wt = _store(q, N, K, seed=100 + M)
    cols = np.random.default_rng(M).choice(K, M, replace=False)
    X = torch.zeros(M, K, dtype=torch.bfloat16)
    X[np.arange(M), cols] = 1.0
    got = _forward(q, w, X.cuda(), r, N, K)
    want = o.bf16_bits(Wt[:, cols].T.astype(np.float32))
    assert np.array_equal(got, want), f"{(got != want).sum()} outputs differ from W~"


@pytest.mark.parametrize("M,K", [(1, 256), (1, 8192), (4, 2048), (16, 1024), (40, 256), (64, 4096)])
def test_random_rows_within_fp32_accumulation(q, M, K):
    N, r = 768, 16
    w, Wt = _store(q, N, K, seed=K + M)
    Xf = torch.randn(M, K).bfloat16()
    got = _bits_to_f64(_forward(q, w, Xf.cuda(), r, N, K))
    X = Xf.double().numpy()
    exact = X @ Wt.T
    e = (K + 16) * 2.0 ** -24 * (np.abs(X) @ np.abs(Wt).T)
    lo = _bits_to_f64(o.bf16_rne_f64(exact - e))
    hi = _bits_to_f64(o.bf16_rne_f64(exact + e))
    inside = (got >= lo) & (got <= hi)
    assert inside.all(), f"{(~inside).sum()} of {got.size} outputs outside the accumulation band"
    same = got == _bits_to_f64(o.bf16_rne_f64(exact))
    assert same.mean() >= 0.99, f"only {same.mean():.4f} of outputs equal bf16_rne(X W~^T)"
