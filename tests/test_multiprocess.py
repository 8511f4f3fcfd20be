"""The multi-rank path on CPU (gloo, world size 2): token-sharded data
parallelism with one all-reduce of the adapter gradients gives the
full-batch gradients, and the bench's timing takes the max over ranks."""
from __future__ import annotations

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import nf4_oracle as o


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    rng = np.random.default_rng(0)
    M, N, K, r, g = 12, 16, 64, 8, 2.0
    W = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    Wt = o.dequantize(*o.quantize(W), N, K).astype(np.float64)
    X, A, B, dY = (rng.normal(size=s) for s in ((M, K), (r, K), (N, r), (M, N)))
    sl = slice(rank * M // world, (rank + 1) * M // world)
    _, dA, dB, _ = o.linear_backward(dY[sl], X[sl], Wt, A, B, g)
    tA, tB = torch.from_numpy(dA), torch.from_numpy(dB)
    bench.allreduce_adapter_grads(tA, tB)
    mx = bench._max_over_ranks(float(rank + 1), world)
    if rank == 0:
        _, dA_full, dB_full, _ = o.linear_backward(dY, X, Wt, A, B, g)
        out.put((np.abs(tA.numpy() - dA_full).max(), np.abs(tB.numpy() - dB_full).max(), mx))
    dist.barrier()
    dist.destroy_process_group()


def test_token_sharded_gradients_sum_to_full_batch():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    ea, eb, mx = q.get(timeout=120)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert ea < 1e-10 and eb < 1e-10
    assert mx == 2.0
