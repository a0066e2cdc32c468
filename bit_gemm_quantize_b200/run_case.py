"""Runs one kernel configuration a few times (for profilers and quick timing).

python -m bit_gemm_quantize_b200.run_case --op gemm_is --M 1024 --K 4096 --N 22016 --reps 3

--op: quant | gemm_is | gemm_fs | gemm_w8 (8-bit weight codes) | gemm_asym
(asymmetric token codes).  Inputs come from the seeded workload generator
(tokens moved off zero by +1 for gemm_asym); weights are packed once before
the repetitions.  Prints the mean CUDA-event time per launch.
"""
from __future__ import annotations

import argparse

import torch

import bit_gemm_quantize_b200 as bgq
from bit_gemm_quantize_b200 import workloads


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", default="gemm_is", choices=["quant", "gemm_is", "gemm_fs", "gemm_w8", "gemm_asym"])
    ap.add_argument("--M", type=int, default=1024)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--N", type=int, default=22016)
    ap.add_argument("--group", type=int, default=128)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--out", default="f16")
    a = ap.parse_args()
    dev = torch.device("cuda:0")
    wl = workloads.make_linear(a.M, a.K, a.N if a.op != "quant" else 8, x_dtype="bf16", seed=7)
    xs = wl.x + 1.0 if a.op == "gemm_asym" else wl.x
    x = torch.from_numpy(xs).to(dev).to(torch.bfloat16)
    if a.op == "gemm_asym":
        q, s, z = bgq.quantize_act_per_token_asym(x)
    else:
        q, s = bgq.quantize_act_per_token(x)
    if a.op == "gemm_w8":
        pk = bgq.pack_w8_groupwise(torch.from_numpy(wl.w).to(dev), group=a.group, alpha=None)
    elif a.op != "quant":
        pk = bgq.pack_w4_groupwise(torch.from_numpy(wl.w).to(dev), group=a.group, alpha=1024)
    if a.op == "gemm_asym":
        zc = bgq.w4_zero_point_term(pk["packed"], pk["S"], group=a.group)
    if a.op != "quant":
        path = {"gemm_is": 0, "gemm_asym": 0, "gemm_fs": 1, "gemm_w8": 2}[a.op]
        ws = bgq.gemm_workspace(a.M, a.N, a.K, a.group, path, dev)

    def once():
        if a.op == "quant":
            bgq.quantize_act_per_token(x, q, s)
        elif a.op == "gemm_is":
            bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], pk["alpha"], group=a.group, out=a.out, workspace=ws)
        elif a.op == "gemm_w8":
            bgq.w8a8_gemm_intscale(q, s, pk["w8"], pk["S"], pk["alpha"], group=a.group, out=a.out, workspace=ws)
        elif a.op == "gemm_asym":
            bgq.w4a8_gemm_intscale_asym(q, s, z, pk["packed"], pk["S"], zc, pk["alpha"], group=a.group, out=a.out,
                                        workspace=ws)
        else:
            bgq.w4a8_gemm_floatscale(q, s, pk["packed"], pk["s_g"], group=a.group, out=a.out, workspace=ws)

    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.reps):
        once()
    e1.record()
    torch.cuda.synchronize()
    print(f"{a.op} M={a.M} K={a.K} N={a.N}: {e0.elapsed_time(e1) / a.reps * 1e3:.2f} us per launch "
          f"(device status {bgq.device_status()})")


if __name__ == "__main__":
    main()
