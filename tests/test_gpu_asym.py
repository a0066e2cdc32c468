"""Parity of the asymmetric-activation path (per-token int8 codes with a zero
point, "Quantization" notes, Asymmetric Quantization) with the CPU oracle,
through the C ABI.

Codes, scale bits, zero points, the weight-side zero-point term and the raw
int32 accumulators must match bit for bit; fp16 outputs are held to the
tolerance of the symmetric path (|y - y_ref| <= 4e-3 * max(|y_ref|, tau),
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


def _shifted(M, K, N, seed, offset, dtype):
    """Synthetic activations moved off zero (as after a one-sided activation
    function) and weights; returns the device input and its exact fp32 copy."""
    wl = workloads.make_linear(M, K, N, x_dtype="f32", seed=seed)
    x = (wl.x + np.float32(offset)).astype(np.float32)
    xt = torch.from_numpy(x).to(_dev()).to(dtype)
    return xt, xt.float().cpu().numpy(), wl.w


@pytest.mark.parametrize("M,K,dtype,offset", [
    (1, 1024, torch.bfloat16, 0.75),
    (7, 4096, torch.float32, 2.0),
    (64, 2048, torch.bfloat16, -1.5),
    (300, 1024, torch.float32, 0.25),
])
def test_quantize_asym_bitexact(M, K, dtype, offset):
    xt, x, _ = _shifted(M, K, 8, seed=M + K, offset=offset, dtype=dtype)
    q, s, z = bgq.quantize_act_per_token_asym(xt)
    qr, sr, zr = oracle.quantize_act_per_token_asym(x)
    assert np.array_equal(_bits(s.cpu().numpy()), _bits(sr))
    assert np.array_equal(z.cpu().numpy(), zr)
    assert np.array_equal(q.cpu().numpy(), qr)
    assert bgq.device_status() == 0


def test_quantize_asym_degenerate_rows():
    dev = _dev()
    K = 256
    rng = np.random.default_rng(5)
    x = rng.standard_normal((6, K)).astype(np.float32)
    x[0] = 0.0                      # zero row: s = 0, z = 0, codes 0
    x[1] = 3.25                     # constant row: range widened to [0, 3.25]
    x[2] = -0.5                     # constant negative row
    x[3] = np.abs(x[3]) + 1.0       # range excludes zero: z clips
    x[4, ::2] = 1e-30               # tiny values next to ordinary ones
    q, s, z = bgq.quantize_act_per_token_asym(torch.from_numpy(x).to(dev))
    qr, sr, zr = oracle.quantize_act_per_token_asym(x)
    assert np.array_equal(_bits(s.cpu().numpy()), _bits(sr))
    assert np.array_equal(z.cpu().numpy(), zr)
    assert np.array_equal(q.cpu().numpy(), qr)


@pytest.mark.parametrize("K,N,qmin", [(1024, 264, -7), (4096, 1024, -8), (11008, 128, -7)])
def test_zero_point_term_bitexact(K, N, qmin):
    dev = _dev()
    wl = workloads.make_linear(1, K, N, seed=K + N)
    pk = bgq.pack_w4_groupwise(torch.from_numpy(wl.w).to(dev), group=128, alpha=None, qmin=qmin)
    zc = bgq.w4_zero_point_term(pk["packed"], pk["S"], group=128, colsum_max=pk["colsum_max"],
                                qmin=qmin).cpu().numpy()
    qw, sg = oracle.quantize_groups(wl.w, 128, qmin=None if qmin == -7 else qmin)
    S = oracle.integer_scales(sg, oracle.amplifier_search(sg))
    want = (np.repeat(S.astype(np.int64), 128, axis=0) * qw.astype(np.int64)).sum(axis=0)
    assert np.all(np.abs(want) < 2**31)
    assert np.array_equal(zc.astype(np.int64), want)


ASYM_CASES = [
    # M, K, N, offset: the decode kernel (one to four tokens, its zero-point
    # correction in the output step), token tiles 16, 32, 64 and 128, ragged M
    # and N, split tiles
    (1, 256, 128, 1.0),
    (2, 4096, 1032, 0.5),
    (3, 1152, 264, -0.75),
    (4, 2048, 520, 2.0),
    (1, 4096, 22016, 1.0),
    (5, 1024, 264, 0.5),
    (16, 4096, 1024, 2.0),
    (33, 1024, 256, -1.0),
    (64, 512, 512, 0.75),
    (130, 768, 1032, 1.25),
    (300, 1024, 256, 3.0),
]


def test_zero_point_term_refuses_weights_beyond_the_asymmetric_bound():
    """Integer scales whose column sums are too large for 255-wide token codes
    are refused before anything is launched."""
    dev = _dev()
    w = torch.full((128 * 64, 8), 0.51, device=dev)  # s_g = 0.51/7; S = 149 at alpha 2^11
    pk = bgq.pack_w4_groupwise(w, alpha=1 << 11)  # 127 * 7 * 128 * 64 * 149 = 1.09e9: the symmetric bound holds
    assert pk["colsum_max"] == 64 * 149
    with pytest.raises(bgq.W4A8Error) as e:  # 255 * 7 * 128 * 64 * 149 = 2.18e9 >= 2^31
        bgq.w4_zero_point_term(pk["packed"], pk["S"], group=128, colsum_max=pk["colsum_max"])
    assert e.value.code == 5


@pytest.mark.parametrize("M,K,N,offset", ASYM_CASES)
def test_gemm_asym_parity(M, K, N, offset):
    dev = _dev()
    xt, x, w = _shifted(M, K, N, seed=13 * M + K, offset=offset, dtype=torch.bfloat16)
    q, s, z = bgq.quantize_act_per_token_asym(xt)
    pk = bgq.pack_w4_groupwise(torch.from_numpy(w).to(dev), group=128, alpha=1024)
    zc = bgq.w4_zero_point_term(pk["packed"], pk["S"], group=128)
    ref = oracle.linear_intscale(x, w, group=128, alpha=1024, out="f32", asym=True)
    assert np.all(np.abs(ref["acc"]) < 2**31)
    acc = bgq.w4a8_gemm_intscale_asym(q, s, z, pk["packed"], pk["S"], zc, 1024, group=128, out="i32")
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref["acc"])
    y = bgq.w4a8_gemm_intscale_asym(q, s, z, pk["packed"], pk["S"], zc, 1024, group=128, out="f16")
    _assert_close_f16(y.float().cpu().numpy(), ref["y64"])
    y32 = bgq.w4a8_gemm_intscale_asym(q, s, z, pk["packed"], pk["S"], zc, 1024, group=128, out="f32")
    y32 = y32.cpu().numpy().astype(np.float64)
    tau = 1e-2 * np.sqrt(np.mean(np.square(ref["y64"])))
    assert (np.abs(y32 - ref["y64"]) / np.maximum(np.abs(ref["y64"]), tau)).max() <= 1e-3
    assert bgq.device_status() == 0


def test_gemm_asym_with_zero_points_zero_is_the_symmetric_gemm():
    # z = 0 and any zc: the asymmetric GEMM reduces to w4a8_gemm_intscale
    dev = _dev()
    wl = workloads.make_linear(48, 2048, 640, x_dtype="bf16", seed=77)
    x = torch.from_numpy(np.ascontiguousarray(wl.x)).to(dev).to(torch.bfloat16)
    q, s = bgq.quantize_act_per_token(x)
    pk = bgq.pack_w4_groupwise(torch.from_numpy(wl.w).to(dev), group=128, alpha=1024)
    zc = bgq.w4_zero_point_term(pk["packed"], pk["S"], group=128)
    z0 = torch.zeros(48, dtype=torch.int32, device=dev)
    a = bgq.w4a8_gemm_intscale_asym(q, s, z0, pk["packed"], pk["S"], zc, 1024, out="i32")
    b = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], 1024, out="i32")
    assert torch.equal(a, b)


def test_gemm_asym_ffn_up_shape_sampled():
    # the FFN up-projection shape (K = 4096, N = 22016) at M = 1024, sampled outputs
    dev = _dev()
    M, K, N = 1024, 4096, 22016
    xt, x, w = _shifted(M, K, N, seed=2024, offset=0.5, dtype=torch.bfloat16)
    q, s, z = bgq.quantize_act_per_token_asym(xt)
    pk = bgq.pack_w4_groupwise(torch.from_numpy(w).to(dev), group=128, alpha=1024)
    zc = bgq.w4_zero_point_term(pk["packed"], pk["S"], group=128)
    acc = bgq.w4a8_gemm_intscale_asym(q, s, z, pk["packed"], pk["S"], zc, 1024, out="i32").cpu().numpy()
    qx, _, zr = oracle.quantize_act_per_token_asym(x)
    assert np.array_equal(q.cpu().numpy(), qx) and np.array_equal(z.cpu().numpy(), zr)
    qw, sg = oracle.quantize_groups(w, 128)
    S = oracle.integer_scales(sg, 1024)
    rng = np.random.default_rng(3)
    ms = rng.integers(0, M, 256)
    ns = rng.integers(0, N, 256)
    # (q - z) q_w accumulated per group: the symmetric accumulator at sampled
    # points minus z times the column term, both from the oracle
    sym = oracle.intscale_acc_at(qx, qw, S, ms, ns)
    col = (np.repeat(S[:, ns].astype(np.int64), 128, axis=0) * qw[:, ns].astype(np.int64)).sum(axis=0)
    want = sym - zr[ms].astype(np.int64) * col
    assert np.array_equal(acc[ms, ns].astype(np.int64), want)
