"""Benchmark of the W4A8 Integer-Scale hot path on B200.

Workload (default): the FFN up-projection batch sweep at the kernel shape of
the Integer Scale summary's kernel comparison (§5.2, Fig. 5a / Fig. 6):
K = 4096, N = 22016, group 128, alpha = 1024, bf16 activations,
M in {1, 8, 32, 128, 512, 1024}, fp16 output.  One step = for every M:
per-token int8 quantization of X [M, K] and the integer-scale W4A8 GEMM.
The float-scale GEMM (the comparison path) is timed beside it per M.

Weights are packed once before timing (offline step).  Six packed copies are
rotated, one per M, so every GEMM streams weights that the previous five
GEMMs (>= 225 MB) have evicted from the 126 MB L2.

Prints one JSON line (rank 0).  `--impl reference` times the CPU oracle on a
bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bit_gemm_quantize_b200 import workloads  # noqa: E402

K_DIM, N_DIM, GROUP, ALPHA = 4096, 22016, 128, 1024
SWEEP = workloads.SWEEP_M
METRIC = "W4A8-IntScale GEMM TOPS and HBM GB/s vs M (1-4096); % of roofline on 1 B200"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
# nominal dense int8 : bf16 tensor throughput on B200 (4.5 : 2.25 PFLOP/s)
INT8_PER_BF16 = 2.0


CASE_OPS = ["quant", "gemm_is", "gemm_fs", "gemm_w8", "gemm_asym", "moe"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    # one kernel configuration, launched --reps times (for profilers and quick
    # timing; prints a one-line summary, not the benchmark's JSON line)
    ap.add_argument("--case", choices=CASE_OPS, default=None,
                    help="quant | gemm_is | gemm_fs | gemm_w8 (8-bit weight codes) | gemm_asym (asymmetric tokens)")
    ap.add_argument("--M", type=int, default=1024)
    ap.add_argument("--K", type=int, default=K_DIM)
    ap.add_argument("--N", type=int, default=N_DIM)
    ap.add_argument("--group", type=int, default=GROUP)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--out", default="f16", choices=["f16", "f32", "i32"])
    return ap.parse_args()


def run_case(a):
    """One kernel configuration, --reps launches back to back on the current
    stream.  Inputs come from the seeded workload generator (tokens moved off
    zero by +1 for gemm_asym); weights are packed once before the launches.
    Prints the mean CUDA-event time per launch and the device status."""
    import torch

    import bit_gemm_quantize_b200 as bgq

    dev = torch.device("cuda:0")
    if a.case == "moe":  # the mixture-of-experts layer of the benchmark (routed quantize + grouped call)
        layer = moe_layer(dev, 3000)[0]["routed"]
        layer()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(a.reps):
            layer()
        e1.record()
        torch.cuda.synchronize()
        st = bgq.device_status()
        print(f"moe: {e0.elapsed_time(e1) / a.reps * 1e3:.2f} us per layer (device status {st})")
        return 0 if st == 0 else 1
    wl = workloads.make_linear(a.M, a.K, a.N if a.case != "quant" else 8, x_dtype="bf16", seed=7,
                               group=a.group)
    xs = wl.x + 1.0 if a.case == "gemm_asym" else wl.x
    x = torch.from_numpy(xs).to(dev).to(torch.bfloat16)
    if a.case == "gemm_asym":
        q, s, z = bgq.quantize_act_per_token_asym(x)
    else:
        q, s = bgq.quantize_act_per_token(x)
    if a.case == "gemm_w8":
        pk = bgq.pack_w8_groupwise(torch.from_numpy(wl.w).to(dev), group=a.group, alpha=None)
    elif a.case != "quant":
        pk = bgq.pack_w4_groupwise(torch.from_numpy(wl.w).to(dev), group=a.group, alpha=ALPHA)
    if a.case == "gemm_asym":
        zc = bgq.w4_zero_point_term(pk["packed"], pk["S"], group=a.group, colsum_max=pk["colsum_max"])
    if a.case != "quant":
        path = {"gemm_is": 0, "gemm_asym": 0, "gemm_fs": 1, "gemm_w8": 2}[a.case]
        ws = bgq.gemm_workspace(a.M, a.N, a.K, a.group, path, dev)

    def once():
        if a.case == "quant":
            bgq.quantize_act_per_token(x, q, s)
        elif a.case == "gemm_is":
            bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], pk["alpha"], group=a.group, out=a.out, workspace=ws)
        elif a.case == "gemm_w8":
            bgq.w8a8_gemm_intscale(q, s, pk["w8"], pk["S"], pk["alpha"], group=a.group, out=a.out, workspace=ws)
        elif a.case == "gemm_asym":
            bgq.w4a8_gemm_intscale_asym(q, s, z, pk["packed"], pk["S"], zc, pk["alpha"], group=a.group, out=a.out,
                                        workspace=ws)
        else:
            bgq.w4a8_gemm_floatscale(q, s, pk["packed"], pk["s_g"], group=a.group,
                                     out="f16" if a.out == "i32" else a.out, workspace=ws)

    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.reps):
        once()
    e1.record()
    torch.cuda.synchronize()
    st = bgq.device_status()
    print(f"{a.case} M={a.M} K={a.K} N={a.N}: {e0.elapsed_time(e1) / a.reps * 1e3:.2f} us per launch "
          f"(device status {st})")
    return 0 if st == 0 else 1


def config_dict():
    return {
        "workload": "ffn_up_sweep",
        "K": K_DIM,
        "N": N_DIM,
        "M": list(SWEEP),
        "group": GROUP,
        "alpha": ALPHA,
        "x_dtype": "bf16",
        "out": "f16",
        "l2": "inputs larger than L2: 6 packed weight copies (271 MB) rotated, one per M",
        "timing": "step = one CUDA graph of all 12 launches, timed with CUDA events over K replays; "
                  "per-launch times from graphs of 6 back-to-back launches on distinct weight copies, "
                  "median of 5 rounds with the two scale paths in alternating order",
    }


def alg_bytes(M, path="is"):
    """Bytes the method must move for one GEMM: int4 W, group scales, int8 codes,
    token scales, fp16 output."""
    G = K_DIM // GROUP
    scale_bytes = (2 if path == "is" else 4) * G * N_DIM
    return N_DIM * K_DIM // 2 + scale_bytes + M * K_DIM + 4 * M + 2 * M * N_DIM


def alg_ops(M):
    return 2 * M * N_DIM * K_DIM


def quant_bytes(M):
    return 2 * M * K_DIM + M * K_DIM + 4 * M


def load_peaks():
    try:
        with open(PEAKS_PATH) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), float(pk["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = "index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active," \
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown," \
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap"

    def __init__(self, index):
        self.index = index
        self.proc = None
        # raw samples go to BENCH_CLOCKS_DIR (default: the system temp folder);
        # the JSON line carries their summary
        folder = os.environ.get("BENCH_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(folder, f"clocks_rank{index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle leg

class OracleLeg:
    """The oracle, as it stands, on bounded samples of the workload: token rows
    of the batch through per-token quantize + group-wise integer GEMM + rescale
    over the full K x N layer.  The weights are quantized once beforehand
    (the offline step, untimed)."""

    def __init__(self, seed: int = 1):
        import oracle

        self.oracle = oracle
        wl = workloads.make_linear(1, K_DIM, N_DIM, x_dtype="bf16", seed=seed)
        self.qw, sg = oracle.quantize_groups(wl.w, GROUP)
        self.S = oracle.integer_scales(sg, ALPHA)

    def run(self, rows: int, seed: int, threads: int = 1):
        """Time `rows` token rows through the oracle.  threads > 1 splits the
        rows over host threads, one oracle call per row (the C oracle releases
        the interpreter lock while it runs, so the calls use separate cores)."""
        o = self.oracle
        x = workloads.make_linear(rows, K_DIM, 8, x_dtype="bf16", seed=seed, check_bound=False).x

        def one(lo, hi):
            qx, sa = o.quantize_act_per_token(x[lo:hi])
            acc = o.intscale_acc(qx, self.qw, self.S, GROUP)
            return o.round_output(o.intscale_output(acc, sa, ALPHA), "f16")

        t0 = time.perf_counter()
        if threads <= 1:
            y = one(0, rows)
        else:
            from concurrent.futures import ThreadPoolExecutor

            with ThreadPoolExecutor(max_workers=threads) as ex:
                y = np.concatenate(list(ex.map(lambda m: one(m, m + 1), range(rows))))
        dt = time.perf_counter() - t0
        assert y.shape == (rows, N_DIM)
        return dt


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_oracle_sample(seed: int = 1):
    """The oracle on the host cores: single-threaded on 8 token rows, and on
    every core on as many rows as there are cores (x2, at least 16)."""
    leg = OracleLeg(seed)
    dt1 = leg.run(8, seed + 1)
    cores = host_cores()
    rows_n = max(16, 2 * cores)
    dtn = leg.run(rows_n, seed + 2, threads=cores)
    return {"value": alg_ops(rows_n) / dtn / 1e12, "unit": "TOPS", "cores": cores, "kind": "oracle",
            "single_core_value": alg_ops(8) / dt1 / 1e12,
            "sample": f"{rows_n} token rows x full K={K_DIM}, N={N_DIM} layer on {cores} threads ({dtn:.1f} s); "
                      f"single core: 8 rows ({dt1:.1f} s); per-token quantize + group-wise integer GEMM + "
                      "rescale"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cores = host_cores()
    rows = cores  # one row per core per step
    leg = OracleLeg(1)
    total_t = 0.0
    for i in range(args.warmup + args.steps):
        dt = leg.run(rows, 10 + i, threads=cores)
        if i >= args.warmup:
            total_t += dt
    v = alg_ops(rows) * args.steps / total_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "TOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_t / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8xi4->i64",
        "data": "synthetic", "config": config_dict(),
        "cpu_baseline": {"value": v, "unit": "TOPS", "cores": cores, "kind": "oracle",
                         "sample": f"each step: {rows} token rows x full K={K_DIM}, N={N_DIM} layer through the "
                                   f"oracle (quantize + group-wise integer GEMM + rescale), one row per host "
                                   f"thread on {cores} threads"},
        "e2e": {"value": v, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- int8 tensor peak

def measure_int8_peak(dev, world, iters=20000, reps=5):
    """The int8 tensor-core rate of this GPU, measured: back-to-back
    tcgen05.mma.kind::i8 (128 x 256 x 32, operands in shared memory, one CTA
    per SM, no loads or epilogue), CUDA events around `reps` launches.  Also
    the 128 x 128 shape with the weight operand in TMEM, as the GEMM issues it."""
    import torch

    import bit_gemm_quantize_b200 as bgq

    stream = torch.cuda.current_stream(dev)
    out = {}
    for key, n, a_tmem in (("ss_n256", 256, False), ("ts_n128", 128, True)):
        for _ in range(2):
            bgq.tensor_i8_peak_probe(iters, n, a_tmem, device=dev)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            ops = bgq.tensor_i8_peak_probe(iters, n, a_tmem, device=dev)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = max_over_ranks([e0.elapsed_time(e1) / reps], world, dev)[0]
        out[key] = ops / (ms * 1e-3) / 1e12
    assert bgq.device_status() == 0
    return out


DECODE = dict(K=4096, N=4096, M=[1, 4, 16])


def measure_decode(dev, rank, world, hbm_peak, reps=7):
    """The decode-shaped layer (K = N = 4096, M in {1, 4, 16}): per-launch time
    of the quantize kernel and of the integer- and float-scale GEMMs, from
    graphs of back-to-back launches that rotate over 36 packed weight copies
    (300 MB, more than twice the L2), so every launch streams its weights from
    HBM.  Inputs drawn on the device: weights ~ N(0, 0.02), tokens ~ N(0, 1)
    with 0.5% of the channels x30, alpha = 1024, fp16 output."""
    import torch

    import bit_gemm_quantize_b200 as bgq

    K, N = DECODE["K"], DECODE["N"]
    g = torch.Generator(device=dev)
    g.manual_seed(6000 + rank)
    w = torch.randn((K, N), generator=g, device=dev)
    w.mul_(0.02)
    pk = bgq.pack_w4_groupwise(w, group=GROUP, alpha=ALPHA)
    del w
    R = 36
    copies = [pk["packed"]] + [pk["packed"].clone() for _ in range(R - 1)]
    stream = torch.cuda.current_stream(dev)

    def per_launch_ms(call):
        for i in range(3):
            call(i)
        torch.cuda.synchronize(dev)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            for i in range(R):
                call(i)
        gr.replay()
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            gr.replay()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            ts.append(e0.elapsed_time(e1) / R)
        del gr
        return max_over_ranks([float(np.median(ts))], world, dev)[0]

    row = {}
    for M in DECODE["M"]:
        x = torch.randn((M, K), generator=g, device=dev)
        cols = torch.randperm(K, generator=g, device=dev)[: max(1, K // 200)]
        x[:, cols] *= 30.0
        x = x.to(torch.bfloat16)
        q, s = bgq.quantize_act_per_token(x)
        y = torch.empty((M, N), dtype=torch.float16, device=dev)
        ws = bgq.gemm_workspace(M, N, K, GROUP, 0, dev)
        wsf = bgq.gemm_workspace(M, N, K, GROUP, 1, dev)
        t_q = per_launch_ms(lambda i: bgq.quantize_act_per_token(x, q, s))
        t_is = per_launch_ms(lambda i: bgq.w4a8_gemm_intscale(q, s, copies[i], pk["S"], ALPHA, group=GROUP, out="f16",
                                                              y=y, workspace=ws))
        t_fs = per_launch_ms(lambda i: bgq.w4a8_gemm_floatscale(q, s, copies[i], pk["s_g"], group=GROUP, out="f16",
                                                                y=y, workspace=wsf))
        b = N * K // 2 + 2 * (K // GROUP) * N + M * K + 4 * M + 2 * M * N
        row[f"is_us_M{M}"] = round(t_is * 1e3, 2)
        row[f"fs_us_M{M}"] = round(t_fs * 1e3, 2)
        row[f"quant_us_M{M}"] = round(t_q * 1e3, 2)
        row[f"frac_hbm_M{M}"] = round(b / (t_is * 1e-3) / 1e9 / hbm_peak, 4)
    row["workload"] = "decode_k4096_n4096"
    row["timing"] = "CUDA events over graphs of 36 launches rotating 36 weight copies (300 MB > L2); median of 7"
    return row


FUSED = dict(K=4096, N=[22016, 4096], M=[1])


def measure_fused(dev, rank, world, hbm_peak, reps=7):
    """Decode with the quantize step fused into the layer's kernel
    (w4a8_linear_intscale: bf16 tokens in, fp16 outputs out, one launch)
    against the two-launch pair (quantize_act_per_token, then
    w4a8_gemm_intscale), per layer, from graphs of back-to-back layers that
    rotate over enough packed weight copies (>= 300 MB) to stream every layer's
    weights from HBM.  Inputs drawn on the device as in measure_decode."""
    import torch

    import bit_gemm_quantize_b200 as bgq

    K = FUSED["K"]
    g = torch.Generator(device=dev)
    g.manual_seed(8000 + rank)
    stream = torch.cuda.current_stream(dev)
    row = {}
    for N in FUSED["N"]:
        w = torch.randn((K, N), generator=g, device=dev)
        w.mul_(0.02)
        pk = bgq.pack_w4_groupwise(w, group=GROUP, alpha=ALPHA)
        del w
        R = max(6, int((300 << 20) // (N * K // 2)) + 1)
        copies = [pk["packed"]] + [pk["packed"].clone() for _ in range(R - 1)]

        def per_layer_ms(call):
            for i in range(3):
                call(i)
            torch.cuda.synchronize(dev)
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr):
                for i in range(R):
                    call(i)
            gr.replay()
            ts = []
            for _ in range(reps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                gr.replay()
                e1.record(stream)
                torch.cuda.synchronize(dev)
                ts.append(e0.elapsed_time(e1) / R)
            del gr
            return max_over_ranks([float(np.median(ts))], world, dev)[0]

        for M in FUSED["M"]:
            x = torch.randn((M, K), generator=g, device=dev)
            cols = torch.randperm(K, generator=g, device=dev)[: max(1, K // 200)]
            x[:, cols] *= 30.0
            x = x.to(torch.bfloat16)
            q = torch.empty((M, K), dtype=torch.int8, device=dev)
            s = torch.empty((M,), dtype=torch.float32, device=dev)
            y = torch.empty((M, N), dtype=torch.float16, device=dev)
            ws = bgq.gemm_workspace(M, N, K, GROUP, 0, dev)

            def pair(i):
                bgq.quantize_act_per_token(x, q, s)
                bgq.w4a8_gemm_intscale(q, s, copies[i], pk["S"], ALPHA, group=GROUP, out="f16", y=y, workspace=ws)

            t_f = per_layer_ms(lambda i: bgq.w4a8_linear_intscale(x, copies[i], pk["S"], ALPHA, group=GROUP,
                                                                  out="f16", y=y, workspace=ws))
            t_p = per_layer_ms(pair)
            b = N * K // 2 + 2 * (K // GROUP) * N + 2 * M * K + 2 * M * N
            row[f"fused_us_n{N}_M{M}"] = round(t_f * 1e3, 2)
            row[f"pair_us_n{N}_M{M}"] = round(t_p * 1e3, 2)
            row[f"fused_frac_hbm_n{N}_M{M}"] = round(b / (t_f * 1e-3) / 1e9 / hbm_peak, 4)
        del copies
    row["workload"] = "decode_fused_quantize_k4096"
    row["timing"] = "CUDA events over graphs of back-to-back layers rotating >= 300 MB of weight copies; median of 7"
    return row


# ---------------------------------------------------------------- mixture of experts

MOE = dict(tokens=2048, K=4096, N=14336, experts=8, topk=2)


def measure_moe(dev, rank, world, int8_peak, reps=10):
    """The Mixtral-shaped layer (2048 tokens, 8 experts of W [4096, 14336],
    top-2): quantize the tokens once, gather the routed rows, one integer-scale
    GEMM per expert with one searched amplifier.  Inputs are drawn on the
    device (seeded Philox): weights ~ N(0, 0.02), tokens ~ N(0, 1) in bf16,
    every token routed to 2 distinct experts uniformly.  The 235 MB of packed
    weights exceed the L2, so every layer streams them from HBM."""
    import torch

    import bit_gemm_quantize_b200 as bgq

    layers, meta = moe_layer(dev, 3000 + rank)
    T, K, N, E, topk = MOE["tokens"], MOE["K"], MOE["N"], MOE["experts"], MOE["topk"]
    R, off, alpha = meta["R"], meta["off"], meta["alpha"]
    stream = torch.cuda.current_stream(dev)

    def layer_ms(layer):
        for _ in range(3):
            layer()
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            layer()
        graph.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        del graph
        return max_over_ranks([e0.elapsed_time(e1) / reps], world, dev)[0]

    ms = layer_ms(layers["routed"])
    ms_g = layer_ms(layers["gather"])
    ops = 2.0 * R * N * K
    tops = ops / (ms * 1e-3) / 1e12
    counts = [int(c) for c in np.diff(off)]
    return {"workload": "moe_mixtral_shaped", "tokens": T, "K": K, "N": N, "experts": E, "topk": topk,
            "group": GROUP, "alpha": alpha, "rows_per_expert": ",".join(str(c) for c in counts),
            "us_per_layer": round(ms * 1e3, 2), "tops": round(tops, 2), "frac_int8": round(tops / int8_peak, 4),
            "us_per_layer_row_gather": round(ms_g * 1e3, 2), "launches_per_layer": 3,
            "timing": "CUDA events over graph replays of one layer: the tokens quantized in routed order "
                      "(quantize_act_routed), the grouped setup and one grouped GEMM over all experts reading "
                      "whole-tile row blocks (device routing offsets); row_gather: tokens quantized once, rows "
                      "gathered by index inside the GEMM; weights > L2"}


def moe_layer(dev, seed):
    """Inputs of the Mixtral-shaped layer and a closure that runs it once
    (quantize, then the grouped call over all experts)."""
    import torch

    import bit_gemm_quantize_b200 as bgq

    T, K, N, E, topk = MOE["tokens"], MOE["K"], MOE["N"], MOE["experts"], MOE["topk"]
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    ws = []
    for _ in range(E):
        w = torch.randn((K, N), generator=g, device=dev)
        w.mul_(0.02)
        ws.append(w)
    pk = bgq.pack_moe_experts(ws, group=GROUP, alpha=None)
    del ws, w
    torch.cuda.empty_cache()
    x = torch.randn((T, K), generator=g, device=dev).to(torch.bfloat16)
    route = torch.argsort(torch.rand((T, E), generator=g, device=dev), dim=1)[:, :topk].cpu().numpy()
    ri, off = workloads.route_rows(route, E)
    R = int(off[-1])
    ri_d = torch.from_numpy(ri).to(dev)
    off_d = torch.from_numpy(off).to(dev)
    wp = bgq.device_pointers(pk["packed"], dev)
    sp = bgq.device_pointers(pk["S"], dev)
    q = torch.empty((T, K), dtype=torch.int8, device=dev)
    s = torch.empty((T,), dtype=torch.float32, device=dev)
    y = torch.empty((R, N), dtype=torch.float16, device=dev)
    wsp = bgq.grouped_workspace(E, N, K, GROUP, dev)

    q_r = torch.empty((R, K), dtype=torch.int8, device=dev)
    s_r = torch.empty((R,), dtype=torch.float32, device=dev)

    def gather():
        bgq.quantize_act_per_token(x, q, s)
        bgq.w4a8_gemm_intscale_grouped(q, s, ri_d, off_d, wp, sp, pk["alpha"], group=GROUP, out="f16", y=y,
                                       workspace=wsp, N=N)

    def routed():
        bgq.quantize_act_routed(x, ri_d, q_r, s_r)
        bgq.w4a8_gemm_intscale_grouped(q_r, s_r, None, off_d, wp, sp, pk["alpha"], group=GROUP, out="f16", y=y,
                                       workspace=wsp, N=N)

    return {"routed": routed, "gather": gather}, {"R": R, "off": off, "alpha": pk["alpha"]}


PREFILL = dict(M=4096, shapes=[(4096, 11008), (11008, 4096)])  # (K, N) of the two layers


def measure_prefill(dev, rank, world, int8_peak, reps=10):
    """The prefill-shaped layers (4096 tokens; K=4096, N=11008 and K=11008,
    N=4096): per-token quantize of bf16 tokens with outlier channels, then the
    integer-scale GEMM with fp16 output.  Inputs are drawn on the device
    (seeded Philox: weights ~ N(0, 0.02), tokens ~ N(0, 1) with 0.5% of the
    channels scaled by 30), alpha = 1024.  The two layers are replayed one
    after the other; together they hold about 300 MB, more than the L2."""
    import torch

    import bit_gemm_quantize_b200 as bgq

    M = PREFILL["M"]
    g = torch.Generator(device=dev)
    g.manual_seed(4000 + rank)
    layers = []
    for K, N in PREFILL["shapes"]:
        w = torch.randn((K, N), generator=g, device=dev)
        w.mul_(0.02)
        pk = bgq.pack_w4_groupwise(w, group=GROUP, alpha=1024)
        del w
        x = torch.randn((M, K), generator=g, device=dev)
        cols = torch.randperm(K, generator=g, device=dev)[: max(1, K // 200)]
        x[:, cols] *= 30.0
        x = x.to(torch.bfloat16)
        q = torch.empty((M, K), dtype=torch.int8, device=dev)
        s = torch.empty((M,), dtype=torch.float32, device=dev)
        y = torch.empty((M, N), dtype=torch.float16, device=dev)
        wsp = bgq.gemm_workspace(M, N, K, GROUP, 0, dev)
        layers.append((K, N, x, q, s, pk, y, wsp))
    torch.cuda.empty_cache()

    def run(layer):
        K, N, x, q, s, pk, y, wsp = layer
        bgq.quantize_act_per_token(x, q, s)
        bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], pk["alpha"], group=GROUP, out="f16", y=y, workspace=wsp)

    graphs = []
    for layer in layers:
        for _ in range(3):
            run(layer)
        torch.cuda.synchronize(dev)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            run(layer)
        gr.replay()
        graphs.append(gr)
    stream = torch.cuda.current_stream(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in graphs]
    tot = [0.0 for _ in graphs]
    torch.cuda.synchronize(dev)
    for _ in range(reps):
        for i, gr in enumerate(graphs):
            ev[i][0].record(stream)
            gr.replay()
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        for i in range(len(graphs)):
            tot[i] += ev[i][0].elapsed_time(ev[i][1])
    ms = max_over_ranks([t / reps for t in tot], world, dev)
    del graphs
    out = {}
    for (K, N, *_), t in zip(layers, ms):
        tops = 2.0 * M * N * K / (t * 1e-3) / 1e12
        out[f"us_k{K}_n{N}"] = round(t * 1e3, 2)
        out[f"tops_k{K}_n{N}"] = round(tops, 2)
        out[f"frac_int8_k{K}_n{N}"] = round(tops / int8_peak, 4)
    return {"workload": "prefill_4096", "M": M, "group": GROUP, "alpha": 1024, **out,
            "timing": "CUDA events around graph replays of quantize + integer-scale GEMM, the two layers alternating"}


W8A8 = dict(K=4096, N=22016, M=[1, 32, 1024])


def measure_w8a8(dev, rank, world, hbm_peak, int8_peak, reps=7):
    """The W8A8 variant on the FFN up-projection shape: 8-bit weight codes with
    integer group scales (alpha from the search), per-launch time of the GEMM
    from graphs of six launches alternating two weight copies (90 MB each, so
    every launch streams its weights from HBM).  Inputs drawn on the device."""
    import torch

    import bit_gemm_quantize_b200 as bgq

    K, N = W8A8["K"], W8A8["N"]
    g = torch.Generator(device=dev)
    g.manual_seed(5000 + rank)
    w = torch.randn((K, N), generator=g, device=dev)
    w.mul_(0.02)
    pk = bgq.pack_w8_groupwise(w, group=GROUP, alpha=None)
    del w
    copies = [pk["w8"], pk["w8"].clone()]
    stream = torch.cuda.current_stream(dev)
    rows = {}
    for M in W8A8["M"]:
        x = torch.randn((M, K), generator=g, device=dev).to(torch.bfloat16)
        q, s = bgq.quantize_act_per_token(x)
        y = torch.empty((M, N), dtype=torch.float16, device=dev)
        wsp = bgq.gemm_workspace(M, N, K, GROUP, 2, dev)

        def call(i):
            bgq.w8a8_gemm_intscale(q, s, copies[i % 2], pk["S"], pk["alpha"], group=GROUP, out="f16", y=y,
                                   workspace=wsp)

        for i in range(3):
            call(i)
        torch.cuda.synchronize(dev)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            for i in range(6):
                call(i)
        gr.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(reps):
            gr.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = max_over_ranks([e0.elapsed_time(e1) / (6 * reps)], world, dev)[0]
        del gr
        bytes_ = N * K + 2 * (K // GROUP) * N + M * K + 4 * M + 2 * M * N
        ops = 2.0 * M * N * K
        t = ms * 1e-3
        gbs, tops = bytes_ / t / 1e9, ops / t / 1e12
        bound = "hbm" if bytes_ / (hbm_peak * 1e9) >= ops / (int8_peak * 1e12) else "tensor"
        rows[f"us_M{M}"] = round(ms * 1e3, 2)
        rows[f"frac_M{M}"] = round(gbs / hbm_peak if bound == "hbm" else tops / int8_peak, 4)
        rows[f"bound_M{M}"] = bound
    return {"workload": "w8a8_ffn_up", "K": K, "N": N, "group": GROUP, "alpha": pk["alpha"], **rows,
            "timing": "CUDA events over graphs of six launches alternating two 90 MB weight copies"}


ASYM = dict(K=4096, N=22016, M=[1, 32, 1024])


def measure_asym(dev, rank, world, reps=7):
    """Asymmetric per-token activations (a zero point per token) against the
    symmetric ones on the FFN up-projection shape: per-launch time of the
    quantize kernels and of the two GEMMs (integer scale, alpha = 1024), from
    graphs of six launches rotating over four packed weight copies (180 MB, so
    every launch streams its weights from HBM).  Inputs drawn on the device,
    moved off zero as after a one-sided activation function."""
    import torch

    import bit_gemm_quantize_b200 as bgq

    K, N = ASYM["K"], ASYM["N"]
    g = torch.Generator(device=dev)
    g.manual_seed(7000 + rank)
    w = torch.randn((K, N), generator=g, device=dev)
    w.mul_(0.02)
    pk = bgq.pack_w4_groupwise(w, group=GROUP, alpha=ALPHA)
    del w
    zc = bgq.w4_zero_point_term(pk["packed"], pk["S"], group=GROUP, colsum_max=pk["colsum_max"])
    copies = [pk["packed"]] + [pk["packed"].clone() for _ in range(3)]
    stream = torch.cuda.current_stream(dev)
    rows = {}

    def per_launch_ms(call):
        for i in range(3):
            call(i)
        torch.cuda.synchronize(dev)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            for i in range(6):
                call(i)
        gr.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(reps):
            gr.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        del gr
        return max_over_ranks([e0.elapsed_time(e1) / (6 * reps)], world, dev)[0]

    for M in ASYM["M"]:
        x = torch.randn((M, K), generator=g, device=dev).add_(1.0).to(torch.bfloat16)
        qa, sa, za = bgq.quantize_act_per_token_asym(x)
        qs, ss = bgq.quantize_act_per_token(x)
        y = torch.empty((M, N), dtype=torch.float16, device=dev)
        wsp = bgq.gemm_workspace(M, N, K, GROUP, 0, dev)
        t_qa = per_launch_ms(lambda i: bgq.quantize_act_per_token_asym(x, qa, sa, za))
        t_qs = per_launch_ms(lambda i: bgq.quantize_act_per_token(x, qs, ss))
        t_ga = per_launch_ms(lambda i: bgq.w4a8_gemm_intscale_asym(
            qa, sa, za, copies[i % 4], pk["S"], zc, ALPHA, group=GROUP, out="f16", y=y, workspace=wsp))
        t_gs = per_launch_ms(lambda i: bgq.w4a8_gemm_intscale(
            qs, ss, copies[i % 4], pk["S"], ALPHA, group=GROUP, out="f16", y=y, workspace=wsp))
        rows[f"quant_asym_us_M{M}"] = round(t_qa * 1e3, 2)
        rows[f"quant_sym_us_M{M}"] = round(t_qs * 1e3, 2)
        rows[f"gemm_asym_us_M{M}"] = round(t_ga * 1e3, 2)
        rows[f"gemm_sym_us_M{M}"] = round(t_gs * 1e3, 2)
    return {"workload": "asym_act_ffn_up", "K": K, "N": N, "group": GROUP, "alpha": ALPHA, **rows,
            "timing": "CUDA events over graphs of six launches rotating four 45 MB weight copies"}


# ---------------------------------------------------------------- rank aggregation

def max_over_ranks(times_ms, world, device):
    """Element-wise maximum over all ranks of this rank's device times (ms).

    Every rank calls it in the same order (one collective); with world == 1
    it returns the times unchanged.
    """
    import torch
    import torch.distributed as dist

    vals = torch.tensor([float(t) for t in times_ms], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(vals, op=dist.ReduceOp.MAX)
    return [float(v) for v in vals]


def whole_job_tops(world, ops_per_step_per_rank, steps, max_ms):
    """Whole-job throughput: the work of all ranks over the slowest rank's time.

    Each rank processes its own, equally sized layer (weak scaling).
    """
    return world * ops_per_step_per_rank * steps / (max_ms * 1e-3) / 1e12


# ---------------------------------------------------------------- GPU leg

def run_ours(args):
    import torch
    import torch.distributed as dist

    import bit_gemm_quantize_b200 as bgq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    hbm_peak, bf16_peak, peak_src = load_peaks()
    int8_derived = bf16_peak * INT8_PER_BF16
    probe = measure_int8_peak(dev, world)
    int8_peak = probe["ss_n256"]  # the measured int8 tensor rate: the large-M roofline's denominator

    # ---- inputs (per rank: an independent layer; weak scaling)
    wl = workloads.make_linear(1, K_DIM, N_DIM, x_dtype="bf16", seed=1000 + rank)
    w_dev = torch.from_numpy(wl.w).to(dev)
    pk = bgq.pack_w4_groupwise(w_dev, group=GROUP, alpha=ALPHA)
    del w_dev
    copies = [pk] + [{k: (v.clone() if isinstance(v, torch.Tensor) else v) for k, v in pk.items()}
                     for _ in range(len(SWEEP) - 1)]
    xs, qs, ss, ys, yfs = [], [], [], [], []
    for i, M in enumerate(SWEEP):
        x = workloads.make_linear(M, K_DIM, 8, x_dtype="bf16", seed=2000 + 10 * rank + i).x
        xs.append(torch.from_numpy(x).to(dev).to(torch.bfloat16))
        qs.append(torch.empty((M, K_DIM), dtype=torch.int8, device=dev))
        ss.append(torch.empty((M,), dtype=torch.float32, device=dev))
        ys.append(torch.empty((M, N_DIM), dtype=torch.float16, device=dev))
        yfs.append(torch.empty((M, N_DIM), dtype=torch.float16, device=dev))
    ws = {M: bgq.gemm_workspace(M, N_DIM, K_DIM, GROUP, 0, dev) for M in SWEEP}
    wsf = {M: bgq.gemm_workspace(M, N_DIM, K_DIM, GROUP, 1, dev) for M in SWEEP}
    # one workspace serves all sequential calls: keep the largest
    ws_all = max([w for w in list(ws.values()) + list(wsf.values()) if w is not None],
                 key=lambda t: t.numel(), default=None)
    stream = torch.cuda.current_stream(dev)

    def quant(i):
        bgq.quantize_act_per_token(xs[i], qs[i], ss[i])

    def gemm_is(i, c):
        bgq.w4a8_gemm_intscale(qs[i], ss[i], c["packed"], c["S"], ALPHA, group=GROUP, out="f16", y=ys[i],
                               workspace=ws_all)

    def gemm_fs(i, c):
        bgq.w4a8_gemm_floatscale(qs[i], ss[i], c["packed"], c["s_g"], group=GROUP, out="f16", y=yfs[i],
                                 workspace=ws_all)

    # warm-up through direct calls
    for _ in range(max(3, args.warmup)):
        for i in range(len(SWEEP)):
            quant(i)
            gemm_is(i, copies[i])
            gemm_fs(i, copies[i])
    torch.cuda.synchronize(dev)

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        return g

    # The step: one graph of all its launches (per M: quantize, then the
    # integer-scale GEMM on that M's weight copy).
    def step_body():
        for i in range(len(SWEEP)):
            quant(i)
            gemm_is(i, copies[i])

    step_graph = capture(step_body)
    # Per-launch durations: graphs of R back-to-back launches of one kernel,
    # each GEMM streaming a different weight copy (cold in L2), so that graph
    # launch latency is amortized over R launches.
    R = len(copies)
    rep_graphs = []
    for i in range(len(SWEEP)):
        gq = capture(lambda i=i: [quant(i) for _ in range(R)])
        gi = capture(lambda i=i: [gemm_is(i, copies[(i + r) % R]) for r in range(R)])
        gf = capture(lambda i=i: [gemm_fs(i, copies[(i + r) % R]) for r in range(R)])
        rep_graphs.append((gq, gi, gf))
    stream = torch.cuda.current_stream(dev)
    for _ in range(max(3, args.warmup)):
        step_graph.replay()
    torch.cuda.synchronize(dev)

    # ---- timed region: K steps of the hot path
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    torch.cuda.nvtx.range_push("timed_step")  # lets a profiler select the timed launches alone
    start.record(stream)
    for _ in range(args.steps):
        step_graph.replay()
    stop.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize(dev)
    barrier()
    clocks = sampler.stop()
    total_ms = start.elapsed_time(stop)

    # ---- per-launch durations (outside the step's timed region)
    def per_launch_ms(g, reps=5):
        g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / (reps * R)

    # Five rounds; in each, the integer- and float-scale graphs of one M run
    # back to back, in alternating order from round to round, so that neither
    # path always follows the other.  The median over rounds is kept.
    q_r, g_r, f_r = [], [], []
    for rnd in range(5):
        q_r.append([per_launch_ms(gq) for (gq, _, _) in rep_graphs])
        g_row, f_row = [], []
        for (_, gi, gf) in rep_graphs:
            if rnd % 2 == 0:
                g_row.append(per_launch_ms(gi))
                f_row.append(per_launch_ms(gf))
            else:
                f_row.append(per_launch_ms(gf))
                g_row.append(per_launch_ms(gi))
        g_r.append(g_row)
        f_r.append(f_row)
    q_ms = np.median(np.array(q_r), axis=0, keepdims=True)
    g_ms = np.median(np.array(g_r), axis=0, keepdims=True)
    f_ms = np.median(np.array(f_r), axis=0, keepdims=True)
    del rep_graphs, step_graph

    # ---- end to end through the public API with host buffers
    xh = [x.cpu().pin_memory() for x in xs]
    yh = [torch.empty((M, N_DIM), dtype=torch.float16).pin_memory() for M in SWEEP]
    xd = [torch.empty_like(x) for x in xs]

    # The calls a user makes (public API, host input in, host output back),
    # pipelined the way a serving loop would run them: uploads on one stream,
    # quantize + GEMM on the main stream, downloads on a third, so a layer's
    # download overlaps the next layers' uploads and compute (PCIe carries
    # both directions at once).
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_step():
        up.wait_stream(stream)  # the previous step's compute has read the device inputs
        ev_in = []
        with torch.cuda.stream(up):
            for i in range(len(SWEEP)):
                xd[i].copy_(xh[i], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(up)
                ev_in.append(ev)
        for i, M in enumerate(SWEEP):
            c = copies[i]
            stream.wait_event(ev_in[i])
            bgq.quantize_act_per_token(xd[i], qs[i], ss[i])
            bgq.w4a8_gemm_intscale(qs[i], ss[i], c["packed"], c["S"], ALPHA, group=GROUP, out="f16", y=ys[i],
                                   workspace=ws_all)
            down.wait_stream(stream)
            with torch.cuda.stream(down):
                yh[i].copy_(ys[i], non_blocking=True)
        stream.wait_stream(down)  # the step ends when every output is on the host

    for _ in range(3):
        e2e_step()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = e0.elapsed_time(e1)
    h2d = sum(M * K_DIM * 2 for M in SWEEP)
    d2h = sum(M * N_DIM * 2 for M in SWEEP)

    # ---- aggregate over ranks: max time
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], world, dev)
    ops_step = sum(alg_ops(M) for M in SWEEP)
    value = whole_job_tops(world, ops_step, args.steps, total_ms)
    e2e_value = whole_job_tops(world, ops_step, args.steps, e2e_ms)

    per_m = {}
    sweep = []
    for i, M in enumerate(SWEEP):
        g = float(np.mean(g_ms[:, i])) * 1e3  # us
        f = float(np.mean(f_ms[:, i])) * 1e3
        q = float(np.mean(q_ms[:, i])) * 1e3
        b_is = alg_bytes(M, "is")
        t_hbm = b_is / (hbm_peak * 1e9)
        t_tc = alg_ops(M) / (int8_peak * 1e12)
        bound = "hbm" if t_hbm >= t_tc else "tensor"
        ach_gbs = b_is / (g * 1e-6) / 1e9
        ach_tops = alg_ops(M) / (g * 1e-6) / 1e12
        sweep.append({
            "M": M, "is_us": round(g, 2), "fs_us": round(f, 2), "quant_us": round(q, 2),
            "is_tops": round(ach_tops, 2), "is_gbs": round(ach_gbs, 1),
            "fs_tops": round(alg_ops(M) / (f * 1e-6) / 1e12, 2),
            "bound": bound,
            "frac_hbm": round(ach_gbs / hbm_peak, 4), "frac_int8": round(ach_tops / int8_peak, 4),
            "is_faster_than_fs": g < f,
        })
        per_m[f"is_us_M{M}"] = round(g, 2)
        per_m[f"fs_us_M{M}"] = round(f, 2)
        per_m[f"quant_us_M{M}"] = round(q, 2)
        per_m[f"frac_M{M}"] = round(ach_gbs / hbm_peak if bound == "hbm" else ach_tops / int8_peak, 4)
        per_m[f"bound_M{M}"] = bound
    per_m["is_faster_than_fs_every_M"] = all(r["is_faster_than_fs"] for r in sweep)
    per_m["frac_is"] = "fraction of the HBM copy bandwidth (bound hbm) or of the measured int8 tensor rate (tensor)"
    shares = g_ms.mean(axis=0)
    dom = int(np.argmax(shares))
    Md = SWEEP[dom]
    gd = float(np.mean(g_ms[:, dom])) * 1e-3  # s
    if sweep[dom]["bound"] == "hbm":
        roof = {"bound": "hbm", "achieved": alg_bytes(Md) / gd / 1e9, "peak": hbm_peak, "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": alg_ops(Md) / gd / 1e12, "peak": int8_peak, "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = measured_traffic(Md)
    roof["kernel"] = f"w4a8_gemm_kernel (integer scale), M={Md} launch"
    roof["peak_source"] = (f"int8: measured tcgen05 kind::i8 probe ({int8_peak:.1f} TOPS, 128x256x32 MMAs, "
                           f"operands in shared memory); HBM: {peak_src} copy {hbm_peak} GB/s")
    roof["frac_of_derived_int8"] = (roof["achieved"] / int8_derived) if roof["bound"] == "tensor" else None

    decode = measure_decode(dev, rank, world, hbm_peak)
    fused = measure_fused(dev, rank, world, hbm_peak)
    moe = measure_moe(dev, rank, world, int8_peak)
    prefill = measure_prefill(dev, rank, world, int8_peak)
    w8a8 = measure_w8a8(dev, rank, world, hbm_peak, int8_peak)
    asym = measure_asym(dev, rank, world)

    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i8xi4->i32", "data": "synthetic",
        "config": config_dict(), "per_M": per_m, "roofline": roof, "clocks": clocks,
        "e2e": {"value": e2e_value, "unit": "TOPS", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 2 * len(SWEEP) * args.steps,
        "int8_peak": {"measured_tops": round(int8_peak, 1), "tmem_a_n128_tops": round(probe["ts_n128"], 1),
                      "derived_bf16x2_tops": round(int8_derived, 1)},
        "decode": decode,
        "fused": fused,
        "moe": moe,
        "prefill": prefill,
        "w8a8": w8a8,
        "asym": asym,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_sample()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


# DRAM bytes (read + write) per launch of the integer-scale GEMM, from one
# ncu capture of `bench.py --case gemm_is --M <M>`, valid for the kernel source
# it was taken with (first 16 hex digits of the SHA-256 of the files below).
MEASURED_TRAFFIC = {1024: (55.458560e6 + 15.798784e6, "23a065b6f9858097")}
GEMM_SOURCES = ("gemm_w4a8.cu", "gemm_w4a8.h", "gemm_common.cuh", "sm100_ptx.cuh")


def gemm_source_digest():
    h = hashlib.sha256()
    base = os.path.join(os.path.dirname(os.path.abspath(__file__)), "bit_gemm_quantize_b200", "csrc")
    for name in GEMM_SOURCES:
        with open(os.path.join(base, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(M):
    rec = MEASURED_TRAFFIC.get(M)
    if rec is None:
        return None
    try:
        digest = gemm_source_digest()
    except OSError:
        return None
    return rec[0] if digest == rec[1] else None


def main():
    args = parse()
    if args.case is not None:
        return run_case(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
