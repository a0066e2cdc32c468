"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Integer results -- activation codes, token-scale bits, packed int4 bytes,
group-scale bits, integer scales, the amplifier, raw int32 accumulators --
must match bit for bit.  Floating-point outputs must satisfy
|y - y_ref| <= rtol * max(|y_ref|, tau), tau = 1e-2 * rms(y_ref), with
rtol = 1e-3 for fp32 output and 4e-3 for fp16 output: y_ref is the oracle's
fp64 result, the GPU rounds twice in fp32 before the output rounding.
"""
import dataclasses

import numpy as np
import pytest
import torch

import bit_gemm_quantize_b200 as bgq
import oracle
from bit_gemm_quantize_b200 import workloads

pytestmark = pytest.mark.gpu

RTOL = {"f32": 1e-3, "f16": 4e-3}


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _to_dev_x(x, x_dtype, dev):
    t = torch.from_numpy(np.ascontiguousarray(x)).to(dev)
    return t.to(torch.bfloat16) if x_dtype == "bf16" else t


def _bits(a):
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


def _assert_close(y, y_ref, out):
    y = np.asarray(y, np.float64)
    tau = 1e-2 * np.sqrt(np.mean(np.square(y_ref))) if y_ref.size else 0.0
    tau = max(tau, 1e-30)
    err = np.abs(y - y_ref) / np.maximum(np.abs(y_ref), tau)
    assert err.max(initial=0.0) <= RTOL[out], f"max rel err {err.max():.3e} (rtol {RTOL[out]})"


# ------------------------------------------------------------------ quantize

QUANT_CASES = [
    (16, 1024, "f32"),   # tiny layer's activations
    (1, 4096, "bf16"),   # decode
    (4, 4096, "bf16"),
    (17, 1040, "bf16"),  # ragged: K not a multiple of 128, odd M
    (300, 11008, "bf16"),  # prefill-like long rows, grid-stride over rows
    (5, 48, "f32"),
    (3, 32768, "f32"),   # rows too long for two shared-memory buffers: direct kernel
]


@pytest.mark.parametrize("M,K,x_dtype", QUANT_CASES)
def test_quantize_bitexact(M, K, x_dtype):
    dev = _dev()
    wl = workloads.make_linear(M, K, 8, x_dtype=x_dtype, seed=M * 7 + K)
    q, s = bgq.quantize_act_per_token(_to_dev_x(wl.x, x_dtype, dev))
    qr, sr = oracle.quantize_act_per_token(wl.x)
    assert np.array_equal(q.cpu().numpy(), qr)
    assert np.array_equal(_bits(s.cpu().numpy()), _bits(sr))


def test_quantize_special_rows():
    """Zero rows, exact ties (x/s = k + 1/2 with s = 1), sign symmetry."""
    dev = _dev()
    K = 64
    x = np.zeros((4, K), np.float32)
    x[1, :8] = [127.0, 0.5, 1.5, 2.5, -0.5, -3.5, 126.5, -127.0]
    x[2] = np.linspace(-3, 3, K, dtype=np.float32)
    x[3] = -x[2]
    q, s = bgq.quantize_act_per_token(torch.from_numpy(x).to(dev))
    qr, sr = oracle.quantize_act_per_token(x)
    assert np.array_equal(q.cpu().numpy(), qr)
    assert np.array_equal(_bits(s.cpu().numpy()), _bits(sr))
    assert q.cpu().numpy()[1, :8].tolist() == [127, 0, 2, 2, 0, -4, 126, -127]
    assert not q.cpu().numpy()[0].any() and s.cpu().numpy()[0] == 0


def test_quantize_empty():
    dev = _dev()
    q, s = bgq.quantize_act_per_token(torch.zeros((0, 256), device=dev))
    assert q.shape == (0, 256) and s.shape == (0,)


# ------------------------------------------------------------------ pack

PACK_CASES = [
    (1024, 1024, 128, 1024),
    (1024, 1024, 128, None),  # amplifier search
    (256, 136, 128, 1024),    # ragged N (not a multiple of 128)
    (512, 264, 256, None),    # group 256
    (4096, 4096, 128, 1024),  # decode layer
]


@pytest.mark.parametrize("K,N,group,alpha", PACK_CASES)
def test_pack_bitexact(K, N, group, alpha):
    dev = _dev()
    wl = workloads.make_linear(1, K, N, seed=K + N + group)
    pk = bgq.pack_w4_groupwise(torch.from_numpy(wl.w).to(dev), group=group, alpha=alpha)
    qw, sg = oracle.quantize_groups(wl.w, group)
    a = oracle.amplifier_search(sg) if alpha is None else alpha
    S = oracle.integer_scales(sg, a)
    assert pk["alpha"] == a
    assert np.array_equal(_bits(pk["s_g"].cpu().numpy()), _bits(sg))
    assert np.array_equal(pk["packed"].cpu().numpy(), oracle.pack_int4(qw))
    assert np.array_equal(pk["S"].cpu().numpy().astype(np.int32), S)
    assert pk["colsum_max"] == oracle.scale_colsum_max(S)


@pytest.mark.parametrize("K,N,group,alpha", [(1024, 1024, 128, 1024), (512, 264, 256, None)])
def test_pack_full_range_bitexact(K, N, group, alpha):
    """Weight codes over the full int4 range [-8, 7] (s_g = max|w| / 8)."""
    dev = _dev()
    wl = workloads.make_linear(1, K, N, seed=5 * K + N)
    pk = bgq.pack_w4_groupwise(torch.from_numpy(wl.w).to(dev), group=group, alpha=alpha, qmin=-8)
    qw, sg = oracle.quantize_groups(wl.w, group, qmin=-8)
    assert qw.min() == -8  # the negative extremes use the extra code
    a = oracle.amplifier_search(sg) if alpha is None else alpha
    S = oracle.integer_scales(sg, a)
    assert pk["alpha"] == a
    assert np.array_equal(_bits(pk["s_g"].cpu().numpy()), _bits(sg))
    assert np.array_equal(pk["packed"].cpu().numpy(), oracle.pack_int4(qw))
    assert np.array_equal(pk["S"].cpu().numpy().astype(np.int32), S)


@pytest.mark.parametrize("M,K,N", [(5, 512, 264), (130, 1024, 392)])
def test_gemm_full_range_parity(M, K, N):
    """The GEMMs with weight codes in [-8, 7]: raw accumulators bit-exact."""
    dev = _dev()
    wl = workloads.make_linear(M, K, N, x_dtype="bf16", seed=7 * M + K)
    x = _to_dev_x(wl.x, wl.x_dtype, dev)
    q, s = bgq.quantize_act_per_token(x)
    pk = bgq.pack_w4_groupwise(torch.from_numpy(wl.w).to(dev), group=128, alpha=1024, qmin=-8)
    ref = oracle.linear_intscale(wl.x, wl.w, group=128, alpha=1024, out="f32", qmin=-8)
    acc = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], pk["alpha"], group=128, out="i32")
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref["acc"])
    y = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], pk["alpha"], group=128, out="f16")
    _assert_close(y.float().cpu().numpy(), ref["y64"], "f16")
    yf = bgq.w4a8_gemm_floatscale(q, s, pk["packed"], pk["s_g"], group=128, out="f32").cpu().numpy()
    _assert_close(yf, oracle.floatscale(ref["qx"], ref["s_a"], ref["qw"], ref["s_g"], 128), "f32")
    assert bgq.device_status() == 0


def test_amplifier_search_device():
    dev = _dev()
    rng = np.random.default_rng(0)
    for _ in range(5):
        s = (10.0 ** rng.uniform(-6, 0.5, 5000)).astype(np.float32)
        s[rng.integers(0, 5000, 50)] = 0.0
        assert bgq.w4a8_amplifier_search(torch.from_numpy(s).to(dev)) == oracle.amplifier_search(s)
    assert bgq.w4a8_amplifier_search(torch.zeros(100, device=dev)) == 1
    with pytest.raises(bgq.W4A8Error):
        bgq.w4a8_amplifier_search(torch.full((10,), 1e-12, device=dev))


def test_pack_scale_range_refused():
    """An amplifier that pushes an integer scale past int16 is refused."""
    dev = _dev()
    w = torch.ones((128, 8), device=dev)  # s_g = 1/7; 1/7 * 2^20 > 32767
    with pytest.raises(bgq.W4A8Error) as e:
        bgq.pack_w4_groupwise(w, alpha=1 << 20)
    assert e.value.code == 6


def test_pack_overflow_bound_refused():
    """Large integer scales over many groups break the int32 accumulator bound."""
    dev = _dev()
    w = torch.full((128 * 64, 8), 0.5, device=dev)  # s_g = 0.5/7, S = 4681 at alpha 2^16
    with pytest.raises(bgq.W4A8Error) as e:
        bgq.pack_w4_groupwise(w, alpha=1 << 16)
    assert e.value.code == 5


# ------------------------------------------------------------------ GEMM

def _gpu_layer(wl, dev, group, alpha):
    x = _to_dev_x(wl.x, wl.x_dtype, dev)
    q, s = bgq.quantize_act_per_token(x)
    pk = bgq.pack_w4_groupwise(torch.from_numpy(wl.w).to(dev), group=group, alpha=alpha)
    return q, s, pk


GEMM_CASES = [
    # M, K, N, group
    (1, 256, 128, 128),
    (3, 512, 136, 128),
    (16, 1024, 1024, 128),
    (17, 384, 264, 128),
    (32, 256, 392, 128),
    (33, 1024, 256, 256),
    (64, 512, 512, 512),   # group = K: per-channel
    (65, 256, 1032, 128),
    (100, 768, 264, 128),
    (128, 512, 640, 128),
    (129, 256, 136, 128),
    (300, 1024, 520, 128),
]


@pytest.mark.parametrize("M,K,N,group", GEMM_CASES)
def test_gemm_intscale_parity(M, K, N, group):
    dev = _dev()
    wl = workloads.make_linear(M, K, N, x_dtype="bf16", seed=M + K + N)
    q, s, pk = _gpu_layer(wl, dev, group, 1024)
    ref = oracle.linear_intscale(wl.x, wl.w, group=group, alpha=1024, out="f32")
    assert np.array_equal(q.cpu().numpy(), ref["qx"])
    assert np.array_equal(pk["packed"].cpu().numpy(), ref["packed"])
    acc = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], pk["alpha"], group=group, out="i32")
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref["acc"])
    for out in ("f32", "f16"):
        y = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], pk["alpha"], group=group, out=out)
        _assert_close(y.float().cpu().numpy(), ref["y64"], out)
    assert bgq.device_status() == 0


@pytest.mark.parametrize("M,K,N,group", GEMM_CASES)
def test_gemm_floatscale_parity(M, K, N, group):
    dev = _dev()
    wl = workloads.make_linear(M, K, N, x_dtype="bf16", seed=M + K + N + 1)
    q, s, pk = _gpu_layer(wl, dev, group, 1024)
    qx, sa = oracle.quantize_act_per_token(wl.x)
    qw, sg = oracle.quantize_groups(wl.w, group)
    yref = oracle.floatscale(qx, sa, qw, sg, group)
    for out in ("f32", "f16"):
        y = bgq.w4a8_gemm_floatscale(q, s, pk["packed"], pk["s_g"], group=group, out=out)
        _assert_close(y.float().cpu().numpy(), yref, out)
    # deterministic: the same call twice gives the same bits
    y1 = bgq.w4a8_gemm_floatscale(q, s, pk["packed"], pk["s_g"], group=group, out="f32")
    y2 = bgq.w4a8_gemm_floatscale(q, s, pk["packed"], pk["s_g"], group=group, out="f32")
    assert torch.equal(y1, y2)


def test_gemm_search_alpha_and_tiny_config():
    """The tiny layer (X fp32 [16,1024] with 4 outlier columns x20, W [1024,1024]),
    fixed amplifier and searched amplifier, fp32 output."""
    dev = _dev()
    wl = workloads.make_linear(16, 1024, 1024, x_dtype="f32", n_outliers=4, outlier_scale=20.0, seed=0)
    for alpha in (1024, None):
        q, s, pk = _gpu_layer(wl, dev, 128, alpha)
        ref = oracle.linear_intscale(wl.x, wl.w, alpha=alpha, out="f32")
        assert pk["alpha"] == ref["alpha"]
        acc = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], pk["alpha"], out="i32")
        assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref["acc"])
        y = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], pk["alpha"], out="f32")
        _assert_close(y.cpu().numpy(), ref["y64"], "f32")


@pytest.mark.parametrize("M,K,N", [(8, 4096, 1024), (200, 1024, 512)])
def test_gemm_intscale_rows_beyond_the_shift_free_bound(M, K, N):
    """Output columns whose sum_g |S[g,n]| is too large for accumulating 16 P_g
    without overflow (here columns 64..127 and 300.., weights scaled up) take the
    shifted drain, the others the shift-free one, inside the same tiles and the
    same split tiles: raw accumulators bit-exact either way."""
    dev = _dev()
    wl = workloads.make_linear(M, K, N, x_dtype="bf16", seed=77 + M)
    w = wl.w.copy()
    big = 6.0 if K >= 4096 else 30.0  # enough groups x scale to pass the bound
    w[:, 64:128] *= big
    w[:, 300:] *= big
    wl = dataclasses.replace(wl, w=w)
    q, s, pk = _gpu_layer(wl, dev, 128, 1024)
    colsum = pk["S"].abs().to(torch.int64).sum(0).cpu().numpy()
    limit = (1 << 31) // (128 * 127 * 128)
    assert (colsum[64:128] > limit).all() and (colsum[:64] <= limit).all()  # both drains are exercised
    ref = oracle.linear_intscale(wl.x, wl.w, group=128, alpha=1024, out="f32")
    acc = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], pk["alpha"], group=128, out="i32")
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref["acc"])
    y = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], pk["alpha"], group=128, out="f16")
    _assert_close(y.float().cpu().numpy(), ref["y64"], "f16")
    assert bgq.device_status() == 0


def test_gemm_zero_input_and_empty():
    dev = _dev()
    wl = workloads.make_linear(8, 256, 128, seed=3)
    wl.x[:] = 0
    q, s, pk = _gpu_layer(wl, dev, 128, 1024)
    y = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], pk["alpha"], out="f32")
    assert not y.cpu().numpy().any()
    q0 = torch.zeros((0, 256), dtype=torch.int8, device=dev)
    s0 = torch.zeros((0,), dtype=torch.float32, device=dev)
    y0 = bgq.w4a8_gemm_intscale(q0, s0, pk["packed"], pk["S"], pk["alpha"])
    assert y0.shape == (0, 128)


def test_gemm_workspace_reuse_across_shapes():
    """Split tiles leave the workspace clean: repeated and interleaved calls agree."""
    dev = _dev()
    outs = []
    for (M, K, N) in [(4, 4096, 512), (16, 2048, 1024), (4, 4096, 512)]:
        wl = workloads.make_linear(M, K, N, seed=11)
        q, s, pk = _gpu_layer(wl, dev, 128, 1024)
        a1 = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], pk["alpha"], out="i32")
        a2 = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], pk["alpha"], out="i32")
        assert torch.equal(a1, a2)
        outs.append(a1.cpu().numpy())
        ref = oracle.linear_intscale(wl.x, wl.w, alpha=1024)
        assert np.array_equal(a1.cpu().numpy().astype(np.int64), ref["acc"])
    assert np.array_equal(outs[0], outs[2])


# ------------------------------------------------------------------ full-size configs, sampled

def _sampled_check(M, K, N, dev, seed, n_samples=1500):
    wl = workloads.make_linear(M, K, N, x_dtype="bf16", seed=seed)
    q, s, pk = _gpu_layer(wl, dev, 128, 1024)
    qx, sa = oracle.quantize_act_per_token(wl.x)
    qw, sg = oracle.quantize_groups(wl.w, 128)
    S = oracle.integer_scales(sg, 1024)
    assert np.array_equal(q.cpu().numpy(), qx)
    assert np.array_equal(_bits(s.cpu().numpy()), _bits(sa))
    assert np.array_equal(pk["packed"].cpu().numpy(), oracle.pack_int4(qw))
    assert np.array_equal(pk["S"].cpu().numpy().astype(np.int32), S)
    rng = np.random.default_rng(seed)
    ms = np.concatenate([rng.integers(0, M, n_samples), [0, M - 1, M - 1, 0]])
    ns = np.concatenate([rng.integers(0, N, n_samples), [0, N - 1, 0, N - 1]])
    acc = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], 1024, out="i32").cpu().numpy()
    acc_ref = oracle.intscale_acc_at(qx, qw, S, ms, ns)
    assert np.array_equal(acc[ms, ns].astype(np.int64), acc_ref)
    y = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], 1024, out="f16").float().cpu().numpy()
    y_ref = acc_ref.astype(np.float64) * sa[ms].astype(np.float64) / 1024.0
    _assert_close(y[ms, ns], y_ref, "f16")
    yf = bgq.w4a8_gemm_floatscale(q, s, pk["packed"], pk["s_g"], out="f16").float().cpu().numpy()
    yf_ref = oracle.floatscale_at(qx, sa, qw, sg, ms, ns)
    _assert_close(yf[ms, ns], yf_ref, "f16")


def _rows_parallel(fn, M):
    """fn(lo, hi) -> the oracle's rows lo..hi-1, run over row blocks on host
    threads (the C oracle releases the interpreter lock while it runs) and
    stacked: the same arithmetic, row by row, in less wall time."""
    from concurrent.futures import ThreadPoolExecutor

    blocks = [(lo, min(M, lo + 2)) for lo in range(0, M, 2)]
    with ThreadPoolExecutor(max_workers=min(16, len(blocks))) as ex:
        parts = list(ex.map(lambda b: fn(*b), blocks))
    return np.concatenate(parts, axis=0)


def _full_check(M, K, N, dev, seed):
    """Every element of the layer against the oracle, at the launch
    configuration the benchmark uses: codes, token-scale bits, packed bytes,
    integer scales, all M x N raw accumulators bit-exact; the integer-scale
    and float-scale fp16 outputs within tolerance."""
    wl = workloads.make_linear(M, K, N, x_dtype="bf16", seed=seed)
    q, s, pk = _gpu_layer(wl, dev, 128, 1024)
    qx, sa = oracle.quantize_act_per_token(wl.x)
    qw, sg = oracle.quantize_groups(wl.w, 128)
    S = oracle.integer_scales(sg, 1024)
    oracle.check_worst_case(S, 128)
    assert np.array_equal(q.cpu().numpy(), qx)
    assert np.array_equal(_bits(s.cpu().numpy()), _bits(sa))
    assert np.array_equal(pk["packed"].cpu().numpy(), oracle.pack_int4(qw))
    assert np.array_equal(pk["S"].cpu().numpy().astype(np.int32), S)
    acc_ref = _rows_parallel(lambda lo, hi: oracle.intscale_acc(qx[lo:hi], qw, S, 128), M)
    acc = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], 1024, out="i32").cpu().numpy()
    assert np.array_equal(acc.astype(np.int64), acc_ref)
    y = bgq.w4a8_gemm_intscale(q, s, pk["packed"], pk["S"], 1024, out="f16").float().cpu().numpy()
    _assert_close(y, oracle.intscale_output(acc_ref, sa, 1024), "f16")
    yf_ref = _rows_parallel(lambda lo, hi: oracle.floatscale(qx[lo:hi], sa[lo:hi], qw, sg, 128), M)
    yf = bgq.w4a8_gemm_floatscale(q, s, pk["packed"], pk["s_g"], out="f16").float().cpu().numpy()
    _assert_close(yf, yf_ref, "f16")
    assert bgq.device_status() == 0


@pytest.mark.parametrize("M", [1, 4, 16])
def test_decode_full_size_every_element(M):
    _full_check(M, 4096, 4096, _dev(), seed=100 + M)


@pytest.mark.parametrize("M", [m for m in workloads.SWEEP_M if m <= 32])
def test_ffn_sweep_full_size_every_element(M):
    _full_check(M, 4096, 22016, _dev(), seed=200 + M)


@pytest.mark.parametrize("M", [m for m in workloads.SWEEP_M if m > 32])
def test_ffn_sweep_full_size_sampled(M):
    _sampled_check(M, 4096, 22016, _dev(), seed=200 + M, n_samples=800)


@pytest.mark.parametrize("K,N", [(4096, 11008), (11008, 4096)])
def test_prefill_full_size_sampled(K, N):
    _sampled_check(4096, K, N, _dev(), seed=300 + K, n_samples=600)
