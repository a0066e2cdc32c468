"""The decode-shaped path (M <= 4 tokens, CUDA-core kernel) and the fused
linear entry point against the oracle: raw int32 accumulators bit-exact,
token codes and scales bit-exact when the kernel quantizes them itself, fp
outputs within the tolerance of the other parity tests."""
import numpy as np
import pytest
import torch

import bit_gemm_quantize_b200 as bgq
import oracle
from bit_gemm_quantize_b200 import workloads

pytestmark = pytest.mark.gpu

RTOL = {"f32": 1e-3, "f16": 4e-3}


def _close(y, y_ref, out):
    y = np.asarray(y, np.float64)
    tau = max(1e-2 * np.sqrt(np.mean(np.square(y_ref))), 1e-30)
    err = np.abs(y - y_ref) / np.maximum(np.abs(y_ref), tau)
    assert err.max(initial=0.0) <= RTOL[out], f"max rel err {err.max():.3e}"


CASES = [
    # M, K, N, group: every token count; ragged N (a CTA's last columns past N
    # read zero-filled rows); groups of 128 .. 4096 (one to 32 128-wide blocks
    # per group); K split over 1 .. 16 warps, rings of 1 .. 16 slots; group = K
    # (per channel); a K that is not a power of two (9 and 86 groups); the
    # largest K of the path; the FFN gate/up shape
    (1, 4096, 4096, 128),
    (2, 1024, 136, 128),
    (3, 2048, 1032, 256),
    (4, 4096, 520, 128),
    (1, 1024, 256, 512),
    (2, 8192, 128, 1024),
    (3, 4096, 264, 2048),
    (4, 4096, 392, 4096),
    (4, 1152, 8, 128),
    (2, 11008, 520, 128),
    (3, 16384, 136, 512),
    (1, 16384, 40, 16384),
    (1, 8192, 22016, 128),
    (2, 4096, 22016, 128),
    (4, 4096, 8192, 128),
    # four tokens and 45 MB of weights: past the decode kernel's size rule (tiles)
    (4, 4096, 22016, 128),
]


@pytest.mark.parametrize("M,K,N,group", CASES)
def test_gemv_intscale_and_floatscale(M, K, N, group):
    dev = torch.device("cuda:0")
    wl = workloads.make_linear(M, K, N, x_dtype="bf16", seed=7 * M + K + N, group=group)
    q, s = bgq.quantize_act_per_token(torch.from_numpy(wl.x).to(dev).to(torch.bfloat16))
    pk = bgq.pack_w4_groupwise(torch.from_numpy(wl.w).to(dev), group=group, alpha=1024)
    ref = oracle.linear_intscale(wl.x, wl.w, group=group, alpha=1024, out="f32")
    if M <= 2 or N * K // 2 <= 32 << 20:  # the decode kernel takes no scratch memory
        assert bgq.load().w4a8_gemm_workspace_size(M, N, K, group, 1) == 0
    acc = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], 1024, group=group, out="i32")
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref["acc"])
    for out in ("f32", "f16"):
        y = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], 1024, group=group, out=out)
        _close(y.float().cpu().numpy(), ref["y64"], out)
    qw, sg = oracle.quantize_groups(wl.w, group)
    yf_ref = oracle.floatscale(ref["qx"], ref["s_a"], qw, sg, group)
    for out in ("f32", "f16"):
        yf = bgq.w4a8_gemm_floatscale(q, s, pk["packed"], pk["s_g"], group=group, out=out)
        _close(yf.float().cpu().numpy(), yf_ref, out)
    assert bgq.device_status() == 0


@pytest.mark.parametrize("M,x_dtype", [(1, "bf16"), (3, "f32"), (4, "bf16"), (5, "bf16"), (16, "f32")])
def test_linear_intscale_quantizes_in_the_kernel(M, x_dtype):
    """Tokens in, outputs out: with one token one kernel quantizes the token
    itself (codes and scale bit-exact); with more tokens and the code buffers
    given, the entry point chains the quantizer and the GEMM."""
    dev = torch.device("cuda:0")
    K, N = 4096, 1032
    wl = workloads.make_linear(M, K, N, x_dtype=x_dtype, seed=90 + M)
    x = torch.from_numpy(wl.x).to(dev)
    if x_dtype == "bf16":
        x = x.to(torch.bfloat16)
    pk = bgq.pack_w4_groupwise(torch.from_numpy(wl.w).to(dev), group=128, alpha=1024)
    ref = oracle.linear_intscale(wl.x, wl.w, group=128, alpha=1024, out="f32")
    q = torch.full((M, K), 99, dtype=torch.int8, device=dev)
    s = torch.full((M,), -1.0, dtype=torch.float32, device=dev)
    acc = bgq.w4a8_linear_intscale(x, pk["packed"], pk["S"], 1024, out="i32", q_x=q, s_a=s)
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), ref["qx"])
    assert np.array_equal(s.cpu().numpy().view(np.uint32), ref["s_a"].view(np.uint32))
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref["acc"])
    y = bgq.w4a8_linear_intscale(x, pk["packed"], pk["S"], 1024, out="f16")
    _close(y.float().cpu().numpy(), ref["y64"], "f16")
    assert bgq.device_status() == 0


def test_linear_intscale_special_rows():
    """A zero row (scale 0, codes 0, output 0) beside ordinary rows, fused."""
    dev = torch.device("cuda:0")
    wl = workloads.make_linear(3, 1024, 256, x_dtype="f32", seed=5)
    wl.x[1] = 0.0
    pk = bgq.pack_w4_groupwise(torch.from_numpy(wl.w).to(dev), group=128, alpha=1024)
    ref = oracle.linear_intscale(wl.x, wl.w, group=128, alpha=1024, out="f32")
    acc = bgq.w4a8_linear_intscale(torch.from_numpy(wl.x).to(dev), pk["packed"], pk["S"], 1024, out="i32")
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref["acc"])
    assert not acc[1].any()


@pytest.mark.parametrize("M,K,N,x_dtype", [(3, 4096, 1032, "f32"), (4, 2048, 520, "bf16"), (2, 1152, 264, "f32")])
def test_linear_intscale_one_kernel_without_buffers(M, K, N, x_dtype):
    """Through the C entry point with no code / scale buffers: with up to four
    tokens the one-kernel route runs (it quantizes the tokens in every CTA);
    raw accumulators bit-exact, fp16 outputs within tolerance."""
    import ctypes

    dev = torch.device("cuda:0")
    wl = workloads.make_linear(M, K, N, x_dtype=x_dtype, seed=300 + M)
    x = torch.from_numpy(wl.x).to(dev)
    if x_dtype == "bf16":
        x = x.to(torch.bfloat16)
    pk = bgq.pack_w4_groupwise(torch.from_numpy(wl.w).to(dev), group=128, alpha=1024)
    ref = oracle.linear_intscale(wl.x, wl.w, group=128, alpha=1024, out="f32")
    lib = bgq.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    x_dt = 2 if x_dtype == "bf16" else 0
    for out, dt, tdt in (("i32", 3, torch.int32), ("f16", 1, torch.float16)):
        y = torch.empty((M, N), dtype=tdt, device=dev)
        code = lib.w4a8_linear_intscale(x.data_ptr(), x_dt, M, K, K, pk["packed"].data_ptr(), pk["S"].data_ptr(),
                                        1024, N, 128, y.data_ptr(), dt, None, None, None, 0, stream)
        assert code == 0
        torch.cuda.synchronize()
        if out == "i32":
            assert np.array_equal(y.cpu().numpy().astype(np.int64), ref["acc"])
        else:
            _close(y.float().cpu().numpy(), ref["y64"], "f16")
    assert bgq.device_status() == 0
