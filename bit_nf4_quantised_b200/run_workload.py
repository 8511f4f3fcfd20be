"""Run a few calls of one synthetic workload through the library (for
profilers such as ncu, which want a short process around the kernels).

  python -m bit_nf4_quantised_b200.run_workload --workload NAME [--calls 2]
         [--forward-only | --merge | --quantize | --quantize-many N]

NAME is a key of synthetic.WORKLOADS; for a multi-layer workload only its
first layer runs.  Each call is one forward (and, unless --forward-only, one
backward) of that layer on cuda:0; with --merge, one merge of the layer's
weight and adapter into a bf16 weight instead; with --quantize, one
quantisation of the layer's fp32 weight; with --quantize-many N, one
qlora_quantize_many call over N separate copies of that weight.
"""
from __future__ import annotations

import argparse

import numpy as np
import torch

from . import _lib as q
from . import synthetic as syn


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="llama7b_attn_proj_4096x4096_m4096_r16")
    ap.add_argument("--calls", type=int, default=2)
    ap.add_argument("--forward-only", action="store_true")
    ap.add_argument("--merge", action="store_true")
    ap.add_argument("--quantize", action="store_true")
    ap.add_argument("--quantize-many", type=int, default=0, metavar="N")
    args = ap.parse_args()
    lin = syn.WORKLOADS[args.workload].layers[0]
    if args.quantize:
        rng = np.random.default_rng(lin.seed)
        W = torch.from_numpy(syn.make_weight(lin, rng)).cuda()
        for _ in range(args.calls):
            q.qlora_quantize(W)
        torch.cuda.synchronize()
        print(f"{args.workload}: {args.calls} quantise call(s)")
        return
    if args.quantize_many > 0:
        rng = np.random.default_rng(lin.seed)
        W = torch.from_numpy(syn.make_weight(lin, rng)).cuda()
        jobs = [(W.clone(), q.empty_nf4(lin.N, lin.K)) for _ in range(args.quantize_many)]
        del W
        for _ in range(args.calls):
            q.qlora_quantize_many(jobs)
        torch.cuda.synchronize()
        print(f"{args.workload}: {args.calls} qlora_quantize_many call(s) of {args.quantize_many}")
        return
    d = syn.make_layer(lin, with_grad=not (args.forward_only or args.merge))
    w = q.qlora_quantize(torch.from_numpy(d["W"]).cuda())
    g = {k: v.cuda() for k, v in d.items() if isinstance(v, torch.Tensor)}
    if args.merge:
        out = torch.empty(lin.N, lin.K, dtype=torch.bfloat16, device="cuda")
        for _ in range(args.calls):
            q.qlora_merge(w, g["A"], g["B"], lin.gamma, out=out)
        torch.cuda.synchronize()
        print(f"{args.workload}: {args.calls} merge call(s)")
        return
    ws = q.workspace(lin.M, lin.N, lin.K, lin.r)
    T = torch.empty(lin.M, lin.r, dtype=torch.float32, device="cuda")
    for _ in range(args.calls):
        q.qlora_linear_forward(g["X"], w, g["A"], g["B"], lin.gamma, T_save=T, ws=ws)
        if not args.forward_only:
            q.qlora_linear_backward(g["dY"], g["X"], w, g["A"], g["B"], lin.gamma, T_saved=T,
                                    ws=ws)
    torch.cuda.synchronize()
    err = q.device_error_word(ws)
    print(f"{args.workload}: {args.calls} call(s), device error word {err}")
    if err:
        raise SystemExit(1)


if __name__ == "__main__":
    main()
