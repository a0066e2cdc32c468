"""Parity of the W8A8 variant (8-bit weight codes with integer group scales)
with the CPU oracle, through the C ABI.

The weight codes, group-scale bits, integer scales, the amplifier and the raw
int32 accumulators must match bit for bit; fp16 outputs are held to the same
tolerance as the W4A8 path (|y - y_ref| <= 4e-3 * max(|y_ref|, tau),
tau = 1e-2 * rms(y_ref)).
"""
import numpy as np
import pytest
import torch

import bit_gemm_quantize_b200 as bgq
import oracle
from bit_gemm_quantize_b200 import workloads

pytestmark = pytest.mark.gpu


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _bits(a):
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


def _assert_close_f16(y, y_ref):
    y = np.asarray(y, np.float64)
    tau = max(1e-2 * np.sqrt(np.mean(np.square(y_ref))), 1e-30)
    err = np.abs(y - y_ref) / np.maximum(np.abs(y_ref), tau)
    assert err.max(initial=0.0) <= 4e-3, f"max rel err {err.max():.3e}"


@pytest.mark.parametrize("K,N,alpha", [(1024, 1024, None), (256, 136, 4096), (4096, 512, None)])
def test_pack_w8_bitexact(K, N, alpha):
    dev = _dev()
    wl = workloads.make_linear(1, K, N, seed=3 * K + N)
    pk = bgq.pack_w8_groupwise(torch.from_numpy(wl.w).to(dev), group=128, alpha=alpha)
    qw, sg = oracle.quantize_groups(wl.w, 128, qmax=127)
    a = oracle.amplifier_search(sg) if alpha is None else alpha
    S = oracle.integer_scales(sg, a)
    assert pk["alpha"] == a
    assert np.array_equal(_bits(pk["s_g"].cpu().numpy()), _bits(sg))
    assert np.array_equal(pk["w8"].cpu().numpy(), qw.T)
    assert np.array_equal(pk["S"].cpu().numpy().astype(np.int32), S)
    assert pk["colsum_max"] == oracle.scale_colsum_max(S)


W8_CASES = [
    # M, K, N: token tiles 16, 32, 64 and 128, ragged M and N, several split tiles
    (1, 256, 128),
    (5, 1024, 264),
    (16, 4096, 1024),
    (17, 512, 392),
    (33, 1024, 256),
    (64, 512, 512),
    (130, 768, 1032),
    (300, 1024, 256),
]


@pytest.mark.parametrize("M,K,N", W8_CASES)
def test_w8a8_gemm_parity(M, K, N):
    dev = _dev()
    wl = workloads.make_linear(M, K, N, x_dtype="bf16", seed=11 * M + K)
    x = torch.from_numpy(np.ascontiguousarray(wl.x)).to(dev).to(torch.bfloat16)
    q, s = bgq.quantize_act_per_token(x)
    pk = bgq.pack_w8_groupwise(torch.from_numpy(wl.w).to(dev), group=128, alpha=None)
    ref = oracle.linear_intscale(wl.x, wl.w, group=128, alpha=None, out="f32", wbits=8)
    assert pk["alpha"] == ref["alpha"]
    acc = bgq.w8a8_gemm_intscale(q, s, pk["w8"], pk["S"], pk["alpha"], group=128, out="i32")
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref["acc"])
    y = bgq.w8a8_gemm_intscale(q, s, pk["w8"], pk["S"], pk["alpha"], group=128, out="f16")
    _assert_close_f16(y.float().cpu().numpy(), ref["y64"])
    assert bgq.device_status() == 0


# One to four tokens take the CUDA-core decode kernel (8-bit codes straight
# from the ring, no unpack): ragged N, K with an odd number of 128-wide blocks,
# the largest K, groups wider than a block, and four tokens on either side of
# the weight-size rule that sends them to the tiles.
W8_DECODE_CASES = [
    # M, K, N, group
    (1, 11008, 4096, 128),
    (2, 1152, 264, 128),
    (3, 4096, 1032, 256),
    (4, 2048, 520, 512),
    (2, 16384, 256, 128),
    (4, 4096, 8192, 128),
    (4, 4096, 8200, 128),
]


@pytest.mark.parametrize("M,K,N,group", W8_DECODE_CASES)
def test_w8a8_decode_parity(M, K, N, group):
    dev = _dev()
    wl = workloads.make_linear(M, K, N, x_dtype="bf16", seed=7 * M + K + N)
    x = torch.from_numpy(np.ascontiguousarray(wl.x)).to(dev).to(torch.bfloat16)
    q, s = bgq.quantize_act_per_token(x)
    pk = bgq.pack_w8_groupwise(torch.from_numpy(wl.w).to(dev), group=group, alpha=None)
    ref = oracle.linear_intscale(wl.x, wl.w, group=group, alpha=None, out="f32", wbits=8)
    assert pk["alpha"] == ref["alpha"]
    if M <= 2 or N * K <= 32 << 20:  # the decode kernel: no workspace
        assert bgq.gemm_workspace(M, N, K, group, 2, dev) is None
    acc = bgq.w8a8_gemm_intscale(q, s, pk["w8"], pk["S"], pk["alpha"], group=group, out="i32")
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref["acc"])
    y = bgq.w8a8_gemm_intscale(q, s, pk["w8"], pk["S"], pk["alpha"], group=group, out="f32")
    _assert_close_f16(y.cpu().numpy(), ref["y64"])
    assert bgq.device_status() == 0


def test_w8a8_matches_dense_integer_product():
    # acc = qx @ (S * q) as one dense integer matmul, at a size with many split tiles
    dev = _dev()
    M, K, N = 8, 4096, 2048
    wl = workloads.make_linear(M, K, N, x_dtype="bf16", seed=99)
    x = torch.from_numpy(np.ascontiguousarray(wl.x)).to(dev).to(torch.bfloat16)
    q, s = bgq.quantize_act_per_token(x)
    pk = bgq.pack_w8_groupwise(torch.from_numpy(wl.w).to(dev), group=128, alpha=None)
    acc = bgq.w8a8_gemm_intscale(q, s, pk["w8"], pk["S"], pk["alpha"], group=128, out="i32").cpu().numpy()
    Wint = np.repeat(pk["S"].cpu().numpy().astype(np.int64), 128, axis=0) * pk["w8"].cpu().numpy().T.astype(np.int64)
    assert np.array_equal(acc.astype(np.int64), q.cpu().numpy().astype(np.int64) @ Wint)


@pytest.mark.parametrize("M", [1, 32, 1024])
def test_w8a8_ffn_up_full_size_sampled(M):
    # the FFN up-projection shape the benchmark times (K = 4096, N = 22016), sampled outputs
    dev = _dev()
    K, N = 4096, 22016
    wl = workloads.make_linear(M, K, N, x_dtype="bf16", seed=400 + M)
    x = torch.from_numpy(np.ascontiguousarray(wl.x)).to(dev).to(torch.bfloat16)
    q, s = bgq.quantize_act_per_token(x)
    pk = bgq.pack_w8_groupwise(torch.from_numpy(wl.w).to(dev), group=128, alpha=None)
    qx, sa = oracle.quantize_act_per_token(wl.x)
    qw, sg = oracle.quantize_groups(wl.w, 128, qmax=127)
    alpha = oracle.amplifier_search(sg)
    S = oracle.integer_scales(sg, alpha)
    assert pk["alpha"] == alpha
    assert np.array_equal(q.cpu().numpy(), qx)
    assert np.array_equal(pk["S"].cpu().numpy().astype(np.int32), S)
    rng = np.random.default_rng(M)
    ms = np.concatenate([rng.integers(0, M, 600), [0, M - 1]])
    ns = np.concatenate([rng.integers(0, N, 600), [0, N - 1]])
    acc = bgq.w8a8_gemm_intscale(q, s, pk["w8"], pk["S"], alpha, group=128, out="i32").cpu().numpy()
    acc_ref = oracle.intscale_acc_at(qx, qw, S, ms, ns)
    assert np.array_equal(acc[ms, ns].astype(np.int64), acc_ref)
    y = bgq.w8a8_gemm_intscale(q, s, pk["w8"], pk["S"], alpha, group=128, out="f16").float().cpu().numpy()
    y_ref = acc_ref.astype(np.float64) * sa[ms].astype(np.float64) / alpha
    _assert_close_f16(y[ms, ns], y_ref)
    assert bgq.device_status() == 0
