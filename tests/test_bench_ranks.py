"""Host-side multi-rank logic of bench.py on CPU: two gloo ranks, each with its
own device time; both must see the maximum, and the whole-job value must
count both ranks' work over the slowest rank's time (weak scaling)."""
import importlib.util
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench = _bench()
        mine = [10.0 + 5.0 * rank, 20.0 - 3.0 * rank]
        got = bench.max_over_ranks(mine, world, "cpu")
        q.put((rank, got, bench.whole_job_tops(world, 1e12, 4, got[0])))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_and_whole_job_value_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=100) for _ in range(world)]
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for _, got, value in results:
        assert got == [15.0, 20.0]  # rank 1's 15 ms step time, rank 0's 20 ms e2e time
        # 2 ranks x 1e12 ops x 4 steps over 15 ms = 533.33 TOPS
        assert value == pytest.approx(2 * 1e12 * 4 / 15e-3 / 1e12)


def test_single_rank_is_identity():
    bench = _bench()
    assert bench.max_over_ranks([3.0, 4.0], 1, "cpu") == [3.0, 4.0]
    assert bench.whole_job_tops(1, 2e12, 10, 20.0) == pytest.approx(2e12 * 10 / 20e-3 / 1e12)


def test_reference_arm_prints_the_contract_line():
    # the reference arm (the oracle on the host cores) needs no GPU: one short
    # run must print one JSON line with the keys the benchmark contract names
    import json
    import subprocess
    import sys

    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["config"]["workload"] == "ffn_up_sweep"
    for k in ("value", "unit", "cores", "kind", "sample"):
        assert k in line["cpu_baseline"], k
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
