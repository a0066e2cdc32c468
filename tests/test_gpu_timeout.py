"""The kernels' bounded waits, made to run out on purpose: with a wait limit
of a few hundred cycles the GEMM gives up instead of waiting for its
pipeline, reports W4A8_ERR_TIMEOUT in the device status word and leaves the
context usable; after the status is cleared (which re-zeroes the workspaces)
the next call is bit-exact against the oracle.  Nothing here faults or hangs
the GPU: every wait that runs out returns, and the copies and MMAs in flight
are waited for at the full limit before the kernel exits."""
import numpy as np
import pytest
import torch

import bit_gemm_quantize_b200 as bgq
import oracle
from bit_gemm_quantize_b200 import workloads

pytestmark = pytest.mark.gpu

W4A8_ERR_TIMEOUT = 8


# 8: 16-token tiles, two CTAs per SM; 300: 128-token tiles with split tiles.
# (The decode kernel's ring waits end within the hardware's own suspend
# window of a blocking try_wait, before the limit is ever checked, so a short
# limit does not make them run out; they report a real stall like the others.)
@pytest.mark.parametrize("M,K,N", [(8, 4096, 2048), (300, 1024, 1032)])
def test_wait_timeout_is_reported_and_the_next_call_is_exact(M, K, N):
    dev = torch.device("cuda:0")
    wl = workloads.make_linear(M, K, N, x_dtype="bf16", seed=31 + M)
    q, s = bgq.quantize_act_per_token(torch.from_numpy(wl.x).to(dev).to(torch.bfloat16))
    pk = bgq.pack_w4_groupwise(torch.from_numpy(wl.w).to(dev), group=128, alpha=1024)
    torch.cuda.synchronize()
    assert bgq.device_status(clear=True) == 0
    lib = bgq.load()
    old = lib.w4a8_set_wait_limit(200)  # SM cycles: far less than a pipeline stage takes
    try:
        timed_out = False
        for _ in range(5):  # a wait that happens to be ready at once cannot run out: try a few launches
            bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], pk["alpha"], out="i32")
            torch.cuda.synchronize()
            st = bgq.device_status(clear=True)  # also re-zeroes the cached workspaces
            assert st in (0, W4A8_ERR_TIMEOUT)
            if st == W4A8_ERR_TIMEOUT:
                timed_out = True
                break
        assert timed_out
    finally:
        lib.w4a8_set_wait_limit(0)
    acc = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], pk["alpha"], out="i32")
    torch.cuda.synchronize()
    assert bgq.device_status() == 0
    ref = oracle.linear_intscale(wl.x, wl.w, group=128, alpha=1024)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref["acc"])


@pytest.mark.parametrize("routed", [True, False])
def test_grouped_wait_timeout_is_reported_and_the_next_call_is_exact(routed):
    """The same for the grouped expert call (setup kernel, then the tiles in
    grouped mode), with rows as blocks of routed-order codes or gathered by
    index."""
    dev = torch.device("cuda:0")
    T, K, N, E = 200, 1024, 520, 3
    wl = workloads.make_moe(T, K, N, E, topk=2, seed=77)
    ri, off = workloads.route_rows(wl.experts, E)
    ri_d = torch.from_numpy(ri.astype(np.int32)).to(dev)
    off_d = torch.from_numpy(np.asarray(off, np.int64)).to(dev)
    x = torch.from_numpy(wl.x).to(dev).to(torch.bfloat16)
    pk = bgq.pack_moe_experts([torch.from_numpy(w).to(dev) for w in wl.w], alpha=1024)
    if routed:
        q, s = bgq.quantize_act_routed(x, ri_d)
        rows = None
    else:
        q, s = bgq.quantize_act_per_token(x)
        rows = ri_d
    ws = bgq.grouped_workspace(E, N, K, 128, dev)

    def call():
        return bgq.w4a8_gemm_intscale_grouped(q, s, rows, off_d, pk["packed"], pk["S"], pk["alpha"], out="i32",
                                              workspace=ws)

    torch.cuda.synchronize()
    assert bgq.device_status(clear=True) == 0
    lib = bgq.load()
    old = lib.w4a8_set_wait_limit(200)
    try:
        timed_out = False
        for _ in range(5):
            call()
            torch.cuda.synchronize()
            st = bgq.device_status(clear=True)
            assert st in (0, W4A8_ERR_TIMEOUT)
            if st == W4A8_ERR_TIMEOUT:
                timed_out = True
                break
        assert timed_out
    finally:
        lib.w4a8_set_wait_limit(0)
    ws.zero_()  # a call that gave up may leave arrival counts in the workspace
    acc = call()
    torch.cuda.synchronize()
    assert bgq.device_status() == 0
    ref = oracle.moe_intscale(wl.x, wl.w, ri, off, alpha=1024)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref["acc"])
