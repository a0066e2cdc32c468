"""Amplifier analysis on the synthetic layers (the analogue of Fig. 4 of the
Integer Scale summary, §4): the amplifier the search picks and its shift count
(Fig. 4(b)), the bits the amplified scales need (Fig. 4(a)), and the weight MSE
between integer-scale and float-scale dequantization for alpha = 2^0 .. 2^14
(Fig. 4(c)).  Oracle-side analysis: CPU only, the seeded synthetic weights.

    python -m oracle.alpha_sweep [--out table.json]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys

import numpy as np

if __package__ in (None, ""):
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle  # noqa: E402
from bit_gemm_quantize_b200 import workloads  # noqa: E402

LAYERS = [("ffn_up K=4096 N=22016", 4096, 22016), ("ffn_down K=11008 N=4096", 11008, 4096)]
ALPHAS = [1 << j for j in range(15)]


def analyse(K: int, N: int, group: int = 128, seed: int = 0) -> dict:
    wl = workloads.make_linear(1, K, N, seed=seed)
    q, s_g = oracle.quantize_groups(wl.w, group)
    alpha = oracle.amplifier_search(s_g)
    S = oracle.integer_scales(s_g, 1024)
    mse, bits = oracle.alpha_sweep(q, s_g, ALPHAS, group=group)
    # float-scale quantization error of the weights themselves, for scale
    deq = q.astype(np.float64) * np.repeat(s_g.astype(np.float64), group, axis=0)
    mse_fs = float(np.mean((deq - wl.w.astype(np.float64)) ** 2))
    return {
        "searched_alpha": int(alpha),
        "shifts": int(round(math.log2(alpha))),
        "S_at_1024_max": int(S.max()),
        "S_at_1024_fraction_below_256": float(np.mean(S < 256)),
        "weight_mse_float_scale_vs_fp32": mse_fs,
        "sweep": [{"alpha": a, "weight_mse_int_vs_float_scale": float(m), "max_S_bits": int(b)}
                  for a, m, b in zip(ALPHAS, mse, bits)],
    }


def main() -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", default=None, help="write the table as JSON")
    args = ap.parse_args()
    table = {}
    for name, K, N in LAYERS:
        r = analyse(K, N)
        table[name] = r
        print(f"{name}: searched alpha 2^{r['shifts']} = {r['searched_alpha']}; at alpha 1024 max S = "
              f"{r['S_at_1024_max']}, {100 * r['S_at_1024_fraction_below_256']:.1f}% of S below 256; "
              f"float-scale weight MSE vs fp32 {r['weight_mse_float_scale_vs_fp32']:.3e}")
        for row in r["sweep"]:
            print(f"  alpha {row['alpha']:6d}: int-vs-float-scale weight MSE {row['weight_mse_int_vs_float_scale']:.3e}"
                  f", largest S needs {row['max_S_bits']} bits")
    if args.out:
        with open(args.out, "w") as f:
            json.dump(table, f, indent=1)
    return 0


if __name__ == "__main__":
    sys.exit(main())
