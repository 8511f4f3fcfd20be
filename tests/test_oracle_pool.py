"""CPU tests of the whole-weight digest helper used by the full-tensor GPU
storage checks: chunking by whole double-quantisation groups gives the same
bytes as one oracle call on the whole tensor, and the spawned pool returns
the same digests."""
from __future__ import annotations

import hashlib

import numpy as np

import _oracle_pool as op
from oracle import nf4_oracle as o
from bit_nf4_quantised_b200 import synthetic as syn


def _direct(W):
    packed, sc, meta = o.quantize(W)
    bits = o.dequantize_bits(packed, sc, meta, W.size)
    return {"packed": hashlib.sha256(packed.tobytes()).hexdigest(),
            "scale_codes": hashlib.sha256(sc.tobytes()).hexdigest(),
            "meta": hashlib.sha256(meta.tobytes()).hexdigest(),
            "wtilde_bits": hashlib.sha256(bits.tobytes()).hexdigest()}


def test_chunked_digests_equal_whole_tensor(monkeypatch):
    W = np.random.default_rng(3).normal(0, 0.02, 16384 * 7 + 64 * 37).astype(np.float32)
    W[5000] = 0.5                                   # a large block somewhere
    monkeypatch.setattr(op, "CHUNK", 16384 * 2)
    assert op._digests_of(W) == _direct(W)


def test_spawned_pool_digest():
    lin = syn.WORKLOADS["single_256x512_m64_r8"].layers[0]
    with op.pool(1) as px:
        got = px.submit(op.oracle_storage_digests, lin).result(timeout=600)
    W = syn.make_weight(lin, np.random.default_rng(lin.seed))
    assert got == _direct(W)
