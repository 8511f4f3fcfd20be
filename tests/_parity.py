"""Shared helpers of the GPU parity tests: oracle-side references built only
from oracle/ and the seeded generators, and the tolerance check of the
layer outputs."""
from __future__ import annotations

import numpy as np
import torch

from oracle import nf4_oracle as o

# Layer-output tolerance: relative Frobenius error and per-element absolute
# error as a fraction of the reference's rms.
REL_FRO = 1e-2
ABS_RMS = 5e-2


def assert_close(name: str, got, ref: np.ndarray) -> dict:
    g = got.detach().to(torch.float64).cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert g.shape == ref.shape, (name, g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{name}: non-finite output"
    nref = np.linalg.norm(ref)
    rms = nref / np.sqrt(max(ref.size, 1))
    diff = g - ref
    rel = np.linalg.norm(diff) / nref if nref > 0 else np.linalg.norm(diff)
    mx = np.abs(diff).max() if diff.size else 0.0
    assert rel <= REL_FRO, f"{name}: relative Frobenius error {rel:.3e} > {REL_FRO}"
    assert mx <= ABS_RMS * rms + 1e-30, f"{name}: max abs error {mx:.3e} > {ABS_RMS} * rms {rms:.3e}"
    return {"rel_fro": float(rel), "max_abs_over_rms": float(mx / rms) if rms > 0 else 0.0}


def oracle_store(W: np.ndarray):
    """(packed, scale_codes, meta) of the oracle for a fp32 weight."""
    return o.quantize(W)


def oracle_wtilde(store, N: int, K: int) -> np.ndarray:
    packed, sc, meta = store
    return o.dequantize(packed, sc, meta, N, K).astype(np.float64)


def groups_of_rows(rows, K: int):
    """Row ranges that cover whole double-quantisation groups (so the oracle
    can quantise just those rows of a big weight and get the same bytes)."""
    per_group = o.BLOCK * o.GROUP
    out = []
    for r in rows:
        e0 = (r * K) // per_group * per_group
        e1 = ((r + 1) * K + per_group - 1) // per_group * per_group
        out.append((e0, e1))
    return out
