"""Seeded synthetic inputs for the QLoRA linear-layer workloads.

Random draws and dtype casts only: nothing of the method's arithmetic lives
here, so both the CUDA path and the CPU oracle can take their inputs from this
module.  Recipe (numpy default_rng, fp32 draws, one generator per layer):

  W   ~ N(0, sigma^2) fp32 [N, K]; if outliers, floor(0.001*N*K) distinct
        positions chosen uniformly are multiplied by 10
  X   ~ N(0, 1) [M, K], rounded to bf16 (round to nearest even)
  A   ~ N(0, 1/K) [r, K] bf16         (LoRA down-projection)
  B   ~ N(0, 0.01^2) [N, r] bf16      (LoRA up-projection; non-zero so the
                                        adapter path is exercised)
  dY  ~ N(0, 1) [M, N] bf16
drawn in that order from default_rng(seed).  gamma = alpha / r.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Linear:
    """One adapted linear layer: W is N x K (out x in), M tokens, rank r."""
    name: str
    M: int
    N: int
    K: int
    r: int
    alpha: float
    sigma: float = 0.02
    outliers: bool = False
    seed: int = 0

    @property
    def gamma(self) -> float:
        return self.alpha / self.r

    def fwd_bwd_flops(self) -> int:
        """Algorithmic flops of forward + dX + dA + dB (T saved, not redone)."""
        M, N, K, r = self.M, self.N, self.K, self.r
        return 4 * M * N * K + 6 * M * r * (N + K)

    def fwd_flops(self) -> int:
        M, N, K, r = self.M, self.N, self.K, self.r
        return 2 * M * N * K + 2 * M * r * (K + N)


@dataclass(frozen=True)
class Workload:
    name: str
    layers: tuple = field(default_factory=tuple)


def _llama7b_decoder(M=4096, r=16, alpha=32, nlayers=32):
    shapes = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
              ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]
    out = []
    for layer in range(nlayers):
        for lid, (nm, N, K) in enumerate(shapes):
            out.append(Linear(f"layer{layer}.{nm}", M, N, K, r, alpha, 0.02, False,
                              1000 * layer + lid))
    return tuple(out)


WORKLOADS = {
    # single small layer, the oracle's full-size parity case
    "single_256x512_m64_r8": Workload("single_256x512_m64_r8", (
        Linear("single", 64, 256, 512, 8, 16.0, 0.02, True, 0),)),
    # Llama-7B attention projection, 4096 tokens (batch 2 x seq 2048)
    "llama7b_attn_proj_4096x4096_m4096_r16": Workload("llama7b_attn_proj_4096x4096_m4096_r16", (
        Linear("attn_proj", 4096, 4096, 4096, 16, 32.0, 0.02, False, 0),)),
    # Llama-7B MLP, 8192 tokens, r = 64 on all three linears
    "llama7b_mlp_m8192_r64": Workload("llama7b_mlp_m8192_r64", (
        Linear("gate", 8192, 11008, 4096, 64, 16.0, 0.02, True, 0),
        Linear("up", 8192, 11008, 4096, 64, 16.0, 0.02, True, 1),
        Linear("down", 8192, 4096, 11008, 64, 16.0, 0.02, True, 2))),
    # decode-shaped GEMV sweep, forward only
    **{f"decode_gemv_{N}x{K}_m{M}": Workload(f"decode_gemv_{N}x{K}_m{M}", (
        Linear(f"gemv_{N}x{K}", M, N, K, 16, 32.0, 0.015, False, 0),))
       for (N, K) in ((28672, 8192), (8192, 28672)) for M in (1, 4, 16)},
    # every linear of a 32-layer Llama-7B-shaped decoder, 4096 tokens
    "llama7b_decoder_32layers_m4096_r16": Workload("llama7b_decoder_32layers_m4096_r16",
                                                    _llama7b_decoder()),
}


def to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def make_weight(lin: Linear, rng: np.random.Generator) -> np.ndarray:
    W = rng.standard_normal((lin.N, lin.K), dtype=np.float32)
    W *= np.float32(lin.sigma)
    if lin.outliers:
        n_out = int(0.001 * lin.N * lin.K)
        pos = rng.choice(lin.N * lin.K, size=n_out, replace=False)
        W.reshape(-1)[pos] *= np.float32(10.0)
    return W


def make_layer(lin: Linear, with_grad: bool = True) -> dict:
    """CPU inputs of one layer: W fp32 numpy; X, A, B, dY bf16 torch tensors."""
    rng = np.random.default_rng(lin.seed)
    W = make_weight(lin, rng)
    X = to_bf16(rng.standard_normal((lin.M, lin.K), dtype=np.float32))
    A = to_bf16(rng.standard_normal((lin.r, lin.K), dtype=np.float32) / np.float32(np.sqrt(lin.K)))
    B = to_bf16(rng.standard_normal((lin.N, lin.r), dtype=np.float32) * np.float32(0.01))
    out = {"W": W, "X": X, "A": A, "B": B, "gamma": lin.gamma}
    if with_grad:
        out["dY"] = to_bf16(rng.standard_normal((lin.M, lin.N), dtype=np.float32))
    return out


def as_f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()
