"""The integer-scale GEMM entry point with the library's fixed per-device
workspace (w4a8_gemm_intscale_static_ws) against the entry point that takes a
caller workspace, on two calls in a row.  Collected last on purpose: it must
pass alone in a fresh process and after every other test.
"""
import pytest
import torch

import bit_gemm_quantize_b200 as bgq
from bit_gemm_quantize_b200 import workloads

pytestmark = pytest.mark.gpu

W4A8_ERR_WORKSPACE = 9


def _inputs(M, K, N, seed):
    dev = torch.device("cuda:0")
    wl = workloads.make_linear(M, K, N, x_dtype="bf16", seed=seed)
    x = torch.from_numpy(wl.x).to(dev).to(torch.bfloat16)
    q, s = bgq.quantize_act_per_token(x)
    pk = bgq.pack_w4_groupwise(torch.from_numpy(wl.w).to(dev), group=128, alpha=1024)
    return q, s, pk


# token tiles 16, 32 and 64, with stream-K partitions that cut tiles (so the
# workspace is used; M = 48 takes the 64-token tile, the widest whose plans fit
# the 8 MiB array), one that cuts none, and a single token (the decode kernel
# needs no workspace; the size reported for it covers the asymmetric-token
# GEMM, which runs tiles even for one token)
@pytest.mark.parametrize("M,K,N,cuts", [(8, 4096, 2048, True), (16, 2048, 1024, True), (32, 4096, 2048, True),
                                        (48, 4096, 2048, True), (16, 128, 256, False), (1, 4096, 2048, True)])
@pytest.mark.parametrize("out", ["i32", "f16"])
def test_static_workspace_matches_caller_workspace(M, K, N, cuts, out):
    need = bgq.load().w4a8_gemm_workspace_size(M, N, K, 128, 0)
    assert (need > 0) == cuts and need <= (8 << 20)
    q, s, pk = _inputs(M, K, N, seed=101 + M)
    ref = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], pk["alpha"], group=128, out=out)
    for _ in range(2):  # two calls in a row: the counters must come back to zero
        got = bgq.w4a8_gemm_intscale_static_ws(q, s, pk["packed"], pk["S"], pk["alpha"], group=128, out=out)
        torch.cuda.synchronize()
        if out == "i32":
            assert torch.equal(got, ref)
        else:
            torch.testing.assert_close(got.float(), ref.float(), rtol=4e-3, atol=1e-2 * ref.float().pow(2).mean().sqrt().item())
    assert bgq.device_status() == 0


def test_static_workspace_refuses_plans_beyond_its_size():
    # token tile 128 with tiles cut across CTAs needs more than the 8 MiB array
    M, K, N = 1024, 4096, 2048
    dev = torch.device("cuda:0")
    assert bgq.load().w4a8_gemm_workspace_size(M, N, K, 128, 0) > (8 << 20)
    q = torch.zeros((M, K), dtype=torch.int8, device=dev)
    s = torch.ones((M,), dtype=torch.float32, device=dev)
    w = torch.zeros((N, K // 2), dtype=torch.uint8, device=dev)
    S = torch.ones((K // 128, N), dtype=torch.int16, device=dev)
    with pytest.raises(bgq.W4A8Error) as e:
        bgq.w4a8_gemm_intscale_static_ws(q, s, w, S, 1024, group=128, out="f16")
    assert e.value.code == W4A8_ERR_WORKSPACE
