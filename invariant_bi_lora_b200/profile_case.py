"""Run one library operation on seeded inputs, for profiler captures.

    python -m invariant_bi_lora_b200.profile_case OP [--M ..] [--K ..] [--N ..]
        [--r ..] [--splits ..] [--mode tree|atomic|unsplit] [--shards ..]
        [--rows ..] [--n ..] [--iters 3]

OP is one of: shrink, shrink_segmented, expand_segmented, gemm, tree_gemm,
rmsnorm, log_softmax, mean.  Inputs are drawn once (seeded) and stay on the
device; the operation runs --iters times back to back.  Meant for
`ncu -k regex:<kernel> -c <n>` on a case whose inputs exceed the L2 cache.
"""
from __future__ import annotations

import argparse

import numpy as np
import torch

from invariant_bi_lora_b200 import bi, synth


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("op")
    ap.add_argument("--M", type=int, default=16384)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--N", type=int, default=4096)
    ap.add_argument("--r", type=int, default=16)
    ap.add_argument("--adapters", type=int, default=8)
    ap.add_argument("--splits", type=int, default=8)
    ap.add_argument("--mode", default="tree")
    ap.add_argument("--shards", type=int, default=8)
    ap.add_argument("--rows", type=int, default=4096)
    ap.add_argument("--n", type=int, default=151936)
    ap.add_argument("--iters", type=int, default=3)
    a = ap.parse_args()
    torch.cuda.set_device(0)

    if a.op in ("shrink", "shrink_segmented", "expand_segmented"):
        d = synth.lora_inputs(a.M, a.K, a.r, n_adapters=a.adapters,
                              N=a.N if a.op == "expand_segmented" else 0, seed=0)
        X, A = dev_bf16(d["x"]), dev_bf16(d["at"])
        y = torch.empty(a.M, a.r, dtype=torch.float32, device="cuda")
        plan = bi.lora_plan(torch.from_numpy(d["ids"]).cuda(), a.adapters)
        if a.op == "shrink":
            run = lambda: bi.lora_shrink(X, A[0].contiguous(), y, a.splits, a.mode)
        elif a.op == "shrink_segmented":
            run = lambda: bi.lora_shrink_segmented(X, A, plan, y, a.splits, a.mode)
        else:
            B = dev_bf16(d["bt"])
            out = torch.empty(a.M, a.N, dtype=torch.float32, device="cuda")
            bi.lora_shrink_segmented(X, A, plan, y, a.splits, "tree")
            run = lambda: bi.lora_expand_segmented(y, B, plan, out)
    elif a.op in ("gemm", "tree_gemm"):
        g_a, g_w = synth.gemm_inputs(a.M, a.N, a.K, seed=0)
        GA, GW = dev_bf16(g_a), dev_bf16(g_w)
        C = torch.empty(a.M, a.N, dtype=torch.float32, device="cuda")
        if a.op == "gemm":
            run = lambda: bi.gemm(GA, GW, C)
        else:
            ws = torch.empty(max(1, bi.gemm_tree_ws_bytes(a.M, a.N, a.shards)), dtype=torch.uint8, device="cuda")
            run = lambda: bi.gemm_tree(GA, GW, C, a.shards, ws)
    elif a.op == "rmsnorm":
        x, w = synth.rmsnorm_inputs(a.rows, a.n, seed=0)
        X, W = dev_bf16(x), dev_bf16(w)
        Y = torch.empty_like(X)
        run = lambda: bi.rmsnorm(X, W, Y)
    elif a.op in ("log_softmax", "mean"):
        X = torch.from_numpy(synth.logits_inputs(a.rows, a.n, seed=0)).cuda()
        if a.op == "log_softmax":
            O = torch.empty_like(X)
            run = lambda: bi.log_softmax(X, O)
        else:
            O = torch.empty(a.rows, dtype=torch.float32, device="cuda")
            run = lambda: bi.mean(X, O)
    else:
        raise SystemExit(f"unknown op {a.op}")

    for _ in range(a.iters):
        run()
    torch.cuda.synchronize()
    st = bi.get_device_status()
    if st != 0:
        raise SystemExit(f"device status {st}")
    print(f"{a.op}: {a.iters} runs ok")


if __name__ == "__main__":
    main()
