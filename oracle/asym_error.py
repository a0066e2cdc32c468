"""Error of symmetric against asymmetric per-token activation codes on the
synthetic layers ("Quantization" notes, Asymmetric Quantization: asymmetric
codes suit activations that are not centred on zero).  Oracle-side analysis:
CPU only, seeded synthetic inputs moved off zero by a constant.

    python -m oracle.asym_error [--out table.json]
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import numpy as np

if __package__ in (None, ""):
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle  # noqa: E402
from bit_gemm_quantize_b200 import workloads  # noqa: E402

OFFSETS = [0.0, 0.5, 1.0, 2.0, 4.0]


def analyse(M: int = 64, K: int = 4096, N: int = 512, seed: int = 0, outliers: bool = True) -> list:
    wl = workloads.make_linear(M, K, N, x_dtype="f32", seed=seed, n_outliers=None if outliers else 0)
    rows = []
    for off in OFFSETS:
        x = (wl.x + np.float32(off)).astype(np.float32)
        exact = x.astype(np.float64) @ wl.w.astype(np.float64)
        rms = float(np.sqrt(np.mean(exact ** 2)))
        ys = oracle.linear_intscale(x, wl.w, alpha=1024, out="f32")
        ya = oracle.linear_intscale(x, wl.w, alpha=1024, out="f32", asym=True)
        qs, ss = oracle.quantize_act_per_token(x)
        qa, sa, za = oracle.quantize_act_per_token_asym(x)
        xs = ss[:, None].astype(np.float64) * qs
        xa = sa[:, None].astype(np.float64) * (qa.astype(np.float64) - za[:, None])
        # the activation codes' share: dequantized tokens against exact weights
        w64 = wl.w.astype(np.float64)
        act_s = float(np.sqrt(np.mean((xs @ w64 - exact) ** 2)) / rms)
        act_a = float(np.sqrt(np.mean((xa @ w64 - exact) ** 2)) / rms)
        rows.append({
            "offset": off,
            "out_rel_rms_err_act_only_sym": act_s,
            "out_rel_rms_err_act_only_asym": act_a,
            "act_mse_sym": float(np.mean((x - xs) ** 2)),
            "act_mse_asym": float(np.mean((x - xa) ** 2)),
            "out_rel_rms_err_sym": float(np.sqrt(np.mean((ys["y64"] - exact) ** 2)) / rms),
            "out_rel_rms_err_asym": float(np.sqrt(np.mean((ya["y64"] - exact) ** 2)) / rms),
        })
    return rows


def main() -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", default=None, help="write the table as JSON")
    args = ap.parse_args()
    table = {}
    for name, outliers in (("with 0.5% outlier channels x30", True), ("no outlier channels", False)):
        rows = analyse(outliers=outliers)
        table[name] = rows
        print(f"{name}: relative rms output error (activation codes only / whole W4A8 layer)")
        print("  offset   symmetric            asymmetric")
        for r in rows:
            print(f"  {r['offset']:6.1f}   {r['out_rel_rms_err_act_only_sym']:.2e} / {r['out_rel_rms_err_sym']:.2e}"
                  f"    {r['out_rel_rms_err_act_only_asym']:.2e} / {r['out_rel_rms_err_asym']:.2e}")
    if args.out:
        with open(args.out, "w") as f:
            json.dump(table, f, indent=1)
    return 0


if __name__ == "__main__":
    sys.exit(main())
