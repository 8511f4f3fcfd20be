"""Whole-weight storage checks: the oracle's quantisation and dequantisation
of a seeded weight, computed in a pool of spawned processes (spawn, so a
worker never inherits a process that has touched the GPU), reduced to SHA-256
digests of the stored bytes and of the dequantised bf16 bits.  The GPU side
hashes the same byte streams in the same order, so equal digests mean every
packed byte, scale code, meta scale and dequantised weight is equal.

The oracle runs on whole double-quantisation groups at a time (16384
weights): groups are independent in the method, so the bytes of a run of
groups are the matching slice of the whole tensor's."""
from __future__ import annotations

import hashlib
import multiprocessing as mp
import os

import numpy as np

CHUNK = 1024 * 64 * 256          # weights per oracle call: 1024 whole groups


def _digests_of(W_flat: np.ndarray) -> dict:
    from oracle import nf4_oracle as o
    h = {k: hashlib.sha256() for k in ("packed", "scale_codes", "meta", "wtilde_bits")}
    for e0 in range(0, W_flat.size, CHUNK):
        part = W_flat[e0:e0 + CHUNK]
        packed, sc, meta = o.quantize(part)
        h["packed"].update(packed.tobytes())
        h["scale_codes"].update(sc.tobytes())
        h["meta"].update(meta.tobytes())
        h["wtilde_bits"].update(o.dequantize_bits(packed, sc, meta, part.size).tobytes())
    return {k: v.hexdigest() for k, v in h.items()}


def oracle_storage_digests(lin) -> dict:
    """Digests of the oracle's stored weight and W~ for a seeded linear."""
    from bit_nf4_quantised_b200 import synthetic as syn
    W = syn.make_weight(lin, np.random.default_rng(lin.seed))
    return _digests_of(W.reshape(-1))


def gpu_storage_digests(w, deq) -> dict:
    """The same digests of a stored weight and its dequantisation on the GPU
    (an NF4Tensor and a bf16 tensor)."""
    def dig(t):
        return hashlib.sha256(t.contiguous().view(-1).cpu().numpy().tobytes()).hexdigest()
    import torch
    return {"packed": dig(w.packed), "scale_codes": dig(w.scale_codes),
            "meta": dig(w.meta_scale.view(torch.int32)),
            "wtilde_bits": dig(deq.view(torch.int16))}


def pool(max_workers: int = 16):
    """A spawn-context process pool sized to the host."""
    from concurrent.futures import ProcessPoolExecutor
    n = max(1, min(max_workers, (os.cpu_count() or 2) - 1))
    return ProcessPoolExecutor(n, mp_context=mp.get_context("spawn"))
