"""Pins for the CPU oracle: each test checks it against something other than
itself -- hand-worked values, closed forms, brute force, library routines on
special cases, and the pages' error model -- chosen so that a dropped term, a
wrong sign, index or transposed operand in the oracle fails at least one.

No GPU is needed here."""
import json
import math
import os

import numpy as np
import pytest

import oracle
from bit_gemm_quantize_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _bits(x):
    return int(np.asarray(x, np.float32).view(np.uint32))


def _nearest_code_bruteforce(x, s, qmax):
    """Search every code for the one nearest to the fp32 quotient x/s, ties to
    the even code.  Uses numpy's fp32 division, independent of the oracle."""
    x = np.asarray(x, np.float32)
    s = np.float32(s)
    if s == 0:
        return np.zeros(x.shape, np.int64)
    t = (x / s).astype(np.float64)  # the quotient, rounded once to fp32
    codes = np.arange(-qmax, qmax + 1, dtype=np.float64)
    d = np.abs(t[..., None] - codes)
    best = d.min(axis=-1, keepdims=True)
    cand = np.where(d == best, codes, np.nan)
    # among equally near codes take the even one
    n_near = (d == best).sum(axis=-1)
    lowest = np.nanmin(cand, axis=-1)
    # a tie has exactly two candidates, one of them even
    tie_pick = np.where(np.fmod(np.abs(lowest), 2) == 0, lowest, lowest + 1)
    return np.where(n_near == 1, lowest, tie_pick).astype(np.int64)


# ------------------------------------------------------------- quantize rows

def test_quantize_golden_rows():
    g = _golden("quantize_int8_symmetric.json")
    for case in g["cases"]:
        q, s = oracle.quantize_act_per_token(np.array([case["x"]], np.float32))
        assert q[0].tolist() == case["q"], case["derivation"]
        assert _bits(s[0]) == int(case["s_bits"], 16), case["derivation"]


def test_quantize_rows_bruteforce_nearest_code():
    rng = np.random.default_rng(1)
    for qmax in (127, 7):
        x = rng.standard_normal((64, 256)).astype(np.float32)
        x[:, 3] *= 20
        q, s = oracle.quantize_rows(x, qmax)
        for m in range(x.shape[0]):
            ref = _nearest_code_bruteforce(x[m], s[m], qmax)
            assert np.array_equal(q[m].astype(np.int64), ref)


def test_quantize_rows_absmax_maps_to_qmax_and_bound():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((32, 512)) * rng.uniform(0.01, 100, (32, 1))).astype(np.float32)
    q, s = oracle.quantize_act_per_token(x)
    am = np.abs(x).max(axis=1)
    arg = np.abs(x).argmax(axis=1)
    # the largest magnitude is the clip point: it lands on +-127
    assert np.all(np.abs(q[np.arange(32), arg]) == 127)
    assert np.all(np.sign(q[np.arange(32), arg]) == np.sign(x[np.arange(32), arg]))
    # s * qmax reproduces the absmax to fp32 rounding
    assert np.allclose(s.astype(np.float64) * 127, am, rtol=2e-7, atol=0)
    # rounding error of a symmetric absmax quantizer: |x - s q| <= s/2 (no clipping)
    err = np.abs(x.astype(np.float64) - s[:, None].astype(np.float64) * q)
    assert np.all(err <= s[:, None] * (0.5 + 1e-5))
    # -128 is never produced
    assert q.min() >= -127 and q.max() <= 127


def test_quantize_rows_error_variance_s2_over_12():
    """Rounding error of a uniform quantizer has variance ~ s^2/12
    (探秘Transformer系列之（34）量化基礎, 量化誤差)."""
    w = workloads.make_linear(64, 4096, 8, x_dtype="f32", seed=3)
    x = w.x
    q, s = oracle.quantize_act_per_token(x)
    mask = np.ones(x.shape[1], bool)
    mask[w.outlier_cols] = False
    e = (x.astype(np.float64) - s[:, None] * q.astype(np.float64))[:, mask]
    ratio = np.mean(e ** 2 / (s[:, None].astype(np.float64) ** 2 / 12.0))
    assert e.size >= 1e5
    assert 0.9 <= ratio <= 1.1, ratio


def test_quantize_zero_row_and_sign_symmetry():
    x = np.array([[0, 0, 0, 0], [1.0, -2.0, 3.0, -4.0]], np.float32)
    q, s = oracle.quantize_act_per_token(x)
    assert s[0] == 0 and not q[0].any()
    qn, sn = oracle.quantize_act_per_token(-x)
    assert np.array_equal(qn, -q) and np.array_equal(sn, s)


# ------------------------------------------------------------- group quantize

def test_quantize_groups_bruteforce_and_layout():
    rng = np.random.default_rng(4)
    K, N, g = 384, 24, 128
    w = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    q, s = oracle.quantize_groups(w, g)
    assert q.shape == (K, N) and s.shape == (K // g, N)
    for gi in range(K // g):
        blk = w[gi * g:(gi + 1) * g]
        # the scale belongs to (group, column): absmax over the group's k only
        assert np.allclose(s[gi].astype(np.float64) * 7, np.abs(blk).max(axis=0), rtol=2e-7)
        for n in range(N):
            ref = _nearest_code_bruteforce(blk[:, n], s[gi, n], 7)
            assert np.array_equal(q[gi * g:(gi + 1) * g, n].astype(np.int64), ref)
    assert q.min() >= -7 and q.max() <= 7


def test_quantize_groups_locality():
    """Changing one weight moves only its own (group, column) scale and codes."""
    rng = np.random.default_rng(5)
    K, N, g = 256, 8, 128
    w = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    q0, s0 = oracle.quantize_groups(w, g)
    w2 = w.copy()
    w2[200, 5] = 1.0
    q1, s1 = oracle.quantize_groups(w2, g)
    diff_s = np.argwhere(s0 != s1)
    assert diff_s.tolist() == [[1, 5]]
    changed = np.argwhere(q0 != q1)
    assert all(128 <= k < 256 and n == 5 for k, n in changed)


def test_quantize_groups_per_channel_equals_rows_of_transpose():
    """group = K is per-channel quantization: the same as per-row of W^T."""
    rng = np.random.default_rng(6)
    w = (rng.standard_normal((256, 16)) * 0.02).astype(np.float32)
    q, s = oracle.quantize_groups(w, 256)
    qt, st = oracle.quantize_rows(w.T.copy(), 7)
    assert np.array_equal(q, qt.T) and np.array_equal(s[0], st)


# ------------------------------------------------------------- packing

def test_pack_golden():
    g = _golden("pack_int4.json")
    q = np.array(g["q_KxN"], np.int8)
    p = oracle.pack_int4(q)
    assert p.tolist() == g["packed_NxK2"], g["derivation"]


def test_pack_exhaustive_nibble_roundtrip():
    vals = np.arange(-8, 8, dtype=np.int8)
    lo, hi = np.meshgrid(vals, vals, indexing="ij")
    rng = np.random.default_rng(11)
    # K=8, N=256: every (code 0, code 4) pair once, the other six codes random
    q = rng.integers(-8, 8, size=(8, 256)).astype(np.int8)
    q[0], q[4] = lo.ravel(), hi.ravel()
    p = oracle.pack_int4(q)
    assert p.shape == (256, 4)
    assert sorted(p[:, 0].tolist()) == list(range(256))  # byte 0 is a bijection of (code 0, code 4)
    assert np.array_equal(oracle.unpack_int4(p, 8, 256), q)
    # nibble semantics: byte j holds code j (low) and code j + 4 (high), two's complement
    for j in range(4):
        b = p[:, j].astype(np.int64)
        assert np.array_equal(((b & 0xF) ^ 8) - 8, q[j])
        assert np.array_equal((((b >> 4) & 0xF) ^ 8) - 8, q[j + 4])
    # the next 8 codes go to the next 4 bytes
    q2 = np.zeros((16, 1), np.int8)
    q2[8:, 0] = np.arange(1, 9)
    assert oracle.pack_int4(q2)[0].tolist() == [0, 0, 0, 0, 0x51, 0x62, 0x73, 0x84]


# ------------------------------------------------------------- amplifier

def test_amplifier_golden():
    for case in _golden("amplifier_search.json")["cases"]:
        assert oracle.amplifier_search(np.array(case["scales"], np.float32)) == case["alpha"], case


def _alpha_closed_form(smin):
    f, e = math.frexp(smin)  # smin = f * 2^e, f in [0.5, 1)
    j = max(0, 1 - e)
    return 1 << j


def test_amplifier_postcondition_and_closed_form():
    rng = np.random.default_rng(7)
    for _ in range(500):
        scales = (10.0 ** rng.uniform(-8, 1, rng.integers(1, 50))).astype(np.float32)
        a = oracle.amplifier_search(scales)
        smin = float(scales.min())
        assert a == _alpha_closed_form(smin)
        assert a >= 1 and (a & (a - 1)) == 0
        assert np.all(scales.astype(np.float64) * a >= 1)
        assert a == 1 or smin * a / 2 < 1


# ------------------------------------------------------------- integer scales

def test_integer_scales_rounding():
    s = np.array([0.0078125, 7.5 / 1024, 8.5 / 1024, 0.0077, 0.005, 0.0], np.float32)
    S = oracle.integer_scales(s, 1024)
    assert S.tolist() == [8, 8, 8, 8, 5, 0]
    rng = np.random.default_rng(8)
    s = rng.uniform(0, 0.05, 10000).astype(np.float32)
    for a in (1, 128, 1024, 4096):
        S = oracle.integer_scales(s, a)
        assert np.all(np.abs(S - s.astype(np.float64) * a) <= 0.5)


# ------------------------------------------------------------- GEMMs

def _rand_codes(rng, M, N, K):
    qx = rng.integers(-127, 128, (M, K)).astype(np.int8)
    qw = rng.integers(-7, 8, (K, N)).astype(np.int8)
    return qx, qw


def test_tiny_linear_golden():
    g = _golden("tiny_linear.json")
    x = np.zeros((1, 256), np.float32)
    w = np.zeros((256, 1), np.float32)
    for k, v in g["x_nonzero"].items():
        x[0, int(k)] = v
    for k, v in g["w_nonzero"].items():
        w[int(k), 0] = v
    r = oracle.linear_intscale(x, w, alpha=1024, out="f32")
    assert r["s_a"].tolist() == [g["s_a"]]
    assert r["s_g"][:, 0].tolist() == g["s_g"]
    assert {str(k): int(r["qx"][0, k]) for k in np.flatnonzero(r["qx"][0])} == g["qx_nonzero"]
    assert {str(k): int(r["qw"][k, 0]) for k in np.flatnonzero(r["qw"][:, 0])} == g["qw_nonzero"]
    assert r["S"][:, 0].tolist() == g["S_alpha1024"]
    assert int(r["acc"][0, 0]) == g["acc_alpha1024"]
    assert r["y64"][0, 0] == g["y"]
    r2 = oracle.linear_intscale(x, w, alpha=None, out="f32")
    assert r2["alpha"] == g["search_alpha"]
    assert r2["S"][:, 0].tolist() == g["S_search"] and int(r2["acc"][0, 0]) == g["acc_search"]
    assert r2["y64"][0, 0] == g["y"]
    f = oracle.linear_floatscale(x, w, out="f32")
    assert f["y64"][0, 0] == g["y"]
    assert float((x.astype(np.float64) @ w.astype(np.float64))[0, 0]) == g["y"]


def test_intscale_groupwise_equals_expanded_weight():
    rng = np.random.default_rng(9)
    for (M, N, K, g) in [(3, 5, 256, 128), (1, 17, 384, 128), (4, 8, 128, 32), (2, 3, 512, 256)]:
        qx, qw = _rand_codes(rng, M, N, K)
        S = rng.integers(-3000, 30000, (K // g, N)).astype(np.int32)
        a = oracle.intscale_acc(qx, qw, S, g)
        b = oracle.intscale_acc_expanded(qx, qw, S, g)
        assert np.array_equal(a, b)
        # and the sampled variant agrees at arbitrary positions
        ms = rng.integers(0, M, 20)
        ns = rng.integers(0, N, 20)
        assert np.array_equal(oracle.intscale_acc_at(qx, qw, S, ms, ns, g), a[ms, ns])


def test_intscale_constant_scale_is_plain_integer_matmul():
    rng = np.random.default_rng(10)
    M, N, K = 6, 11, 512
    qx, qw = _rand_codes(rng, M, N, K)
    Sn = rng.integers(1, 40, N).astype(np.int32)
    S = np.tile(Sn, (K // 128, 1))
    acc = oracle.intscale_acc(qx, qw, S)
    ref = (qx.astype(np.int64) @ qw.astype(np.int64)) * Sn.astype(np.int64)
    assert np.array_equal(acc, ref)


def test_intscale_bruteforce_dequantized_fp64():
    """acc * s_a / alpha equals the fp64 matmul of the dequantized operands
    (s_a q_x) and (S/alpha q_w) on tiny inputs."""
    rng = np.random.default_rng(11)
    for seed in range(300):
        M = int(rng.integers(1, 5))
        N = int(rng.integers(1, 9))
        K = int(rng.choice([128, 256]))
        x = rng.standard_normal((M, K)).astype(np.float32)
        w = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
        alpha = int(rng.choice([1024, 256]))
        r = oracle.linear_intscale(x, w, alpha=alpha, out="f32")
        xh = r["s_a"][:, None].astype(np.float64) * r["qx"]
        G = K // 128
        Sfull = np.repeat(r["S"], 128, axis=0).astype(np.float64)
        wh = Sfull / alpha * r["qw"]
        ref = xh @ wh
        assert np.allclose(r["y64"], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_intscale_zero_input_and_one_hot_column():
    rng = np.random.default_rng(12)
    M, K, N = 3, 256, 4
    w = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    r0 = oracle.linear_intscale(np.zeros((M, K), np.float32), w, out="f32")
    assert not r0["acc"].any() and not r0["y64"].any()
    # one-hot weight column: only k* = 150 (group 1) is non-zero in column 2
    x = rng.standard_normal((M, K)).astype(np.float32)
    w[:, 2] = 0
    w[150, 2] = -0.03
    r = oracle.linear_intscale(x, w, alpha=1024, out="f32")
    S = r["S"][1, 2]
    assert r["qw"][150, 2] == -7 and r["S"][0, 2] == 0
    expect = r["s_a"].astype(np.float64) * S / 1024 * (-7) * r["qx"][:, 150]
    assert np.allclose(r["y64"][:, 2], expect, rtol=1e-15)


def test_floatscale_equals_intscale_when_scales_are_exact():
    """With s_g = S/alpha exactly, the float-scale path must give the
    integer-scale result (two different summations)."""
    rng = np.random.default_rng(13)
    M, N, K = 5, 9, 384
    qx, qw = _rand_codes(rng, M, N, K)
    S = rng.integers(1, 20, (K // 128, N)).astype(np.int32)
    s_a = rng.uniform(0.01, 0.1, M).astype(np.float32)
    s_g = (S / 1024.0).astype(np.float32)
    yf = oracle.floatscale(qx, s_a, qw, s_g)
    yi = oracle.intscale_output(oracle.intscale_acc(qx, qw, S), s_a, 1024)
    assert np.allclose(yf, yi, rtol=1e-12, atol=1e-12)
    ms = np.array([0, 4, 2])
    ns = np.array([8, 0, 3])
    assert np.allclose(oracle.floatscale_at(qx, s_a, qw, s_g, ms, ns), yf[ms, ns], rtol=1e-15)


def test_floatscale_per_channel_is_outer_product_dequant():
    """group = K: y = (s_a s_w^T) o (q_x q_w), the token x channel outer-product
    dequantization (探秘Transformer系列之（34）, 逐通道量化 & 逐token量化)."""
    rng = np.random.default_rng(14)
    M, N, K = 4, 6, 256
    x = rng.standard_normal((M, K)).astype(np.float32)
    w = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    qx, s_a = oracle.quantize_act_per_token(x)
    qw, s_w = oracle.quantize_groups(w, K)
    y = oracle.floatscale(qx, s_a, qw, s_w, K)
    ref = np.outer(s_a.astype(np.float64), s_w[0].astype(np.float64)) * (qx.astype(np.int64) @ qw.astype(np.int64))
    assert np.allclose(y, ref, rtol=1e-14)


def test_intscale_error_bound_against_unquantized():
    """Per element: |y_IS - x w| <= sum_k |x_hat| (s_g/2 + 3.5/alpha) + (s_a/2)|w|,
    from |x - x_hat| <= s_a/2 and |w - (S/alpha) q_w| <= s_g/2 + 7/(2 alpha)."""
    for cfg_seed, (M, K, N) in enumerate([(16, 1024, 64), (4, 512, 96)]):
        wl = workloads.make_linear(M, K, N, x_dtype="f32", seed=cfg_seed, outlier_scale=20.0)
        for alpha in (1024, None):
            r = oracle.linear_intscale(wl.x, wl.w, alpha=alpha, out="f32")
            a = r["alpha"]
            xh = np.abs(r["s_a"][:, None].astype(np.float64) * r["qx"])
            sg = np.repeat(r["s_g"], 128, axis=0).astype(np.float64)
            bound = xh @ (sg / 2 + 3.5 / a) + (r["s_a"][:, None].astype(np.float64) / 2) @ np.ones((1, K)) @ np.abs(wl.w.astype(np.float64))
            y_true = wl.x.astype(np.float64) @ wl.w.astype(np.float64)
            err = np.abs(r["y64"] - y_true)
            assert np.all(err <= bound * (1 + 1e-9) + 1e-12)


def test_int32_bound_and_colsum():
    rng = np.random.default_rng(15)
    K, N = 512, 10
    qx = np.full((2, K), 127, np.int8)
    qw = np.full((K, N), 7, np.int8)
    qx[1] = -127
    S = rng.integers(0, 50, (K // 128, N)).astype(np.int32)
    acc = oracle.intscale_acc(qx, qw, S)
    colsum = oracle.scale_colsum_max(S)
    assert colsum == int(np.abs(S).sum(axis=0).max())
    # extreme codes reach the bound exactly at the column with the largest sum
    assert int(np.abs(acc).max()) == 127 * 7 * 128 * colsum


def test_workload_bound_holds_for_default_amplifier():
    """The generator's weights keep the worst-case accumulator inside int32."""
    wl = workloads.make_linear(1, 4096, 512, seed=0)
    qw, s_g = oracle.quantize_groups(wl.w, 128)
    S = oracle.integer_scales(s_g, 1024)
    assert S.max() <= 32767
    assert 127 * 7 * 128 * oracle.scale_colsum_max(S) < 2 ** 31


def test_oracle_refuses_accumulators_outside_int32():
    """Extreme codes with scales large enough to pass 2^31: the oracle raises
    instead of returning an accumulator the int32 GPU path cannot hold."""
    K, N = 1024, 4
    qx = np.full((1, K), 127, np.int8)
    qw = np.full((K, N), 7, np.int8)
    S = np.full((K // 128, N), 2400, np.int32)  # 127 * 7 * 128 * 8 * 2400 = 2.18e9 > 2^31
    with pytest.raises(oracle.Int32BoundError):
        oracle.intscale_acc(qx, qw, S)
    with pytest.raises(oracle.Int32BoundError):
        oracle.intscale_acc_at(qx, qw, S, [0], [1])
    with pytest.raises(oracle.Int32BoundError):
        oracle.check_worst_case(S, 128)
    S[:] = 2300  # 2.09e9 < 2^31: fine
    acc = oracle.intscale_acc(qx, qw, S)
    assert int(acc.max()) == 127 * 7 * 128 * 8 * 2300
    oracle.check_worst_case(S, 128)


def test_generator_refuses_weights_beyond_the_int32_bound():
    """The seeded generator checks every layer it returns against the worst-case
    accumulator bound (a conservative upper bound from the raw weights)."""
    with pytest.raises(ValueError):
        workloads.make_linear(1, 4096, 64, w_std=2.0, seed=1)  # S ~ 1000 over 32 groups
    with pytest.raises(ValueError):
        workloads.make_moe(4, 4096, 64, 2, w_std=2.0, alpha=1024, seed=1)
    wl = workloads.make_linear(1, 4096, 64, w_std=2.0, seed=1, alpha=None)  # searched amplifier: fine
    # the generator's bound is an upper bound of the exact worst case the oracle computes
    for alpha in (1024, None):
        wl = workloads.make_linear(2, 2048, 96, seed=5, alpha=alpha)
        qw, s_g = oracle.quantize_groups(wl.w, 128)
        a = oracle.amplifier_search(s_g) if alpha is None else alpha
        S = oracle.integer_scales(s_g, a)
        exact = 127 * 7 * 128 * oracle.scale_colsum_max(S)
        upper = workloads.int32_bound_upper(wl.w, 128, alpha)
        assert exact <= upper <= exact * 1.2 + 127 * 7 * 128 * 16


# ------------------------------------------------------------ mixture of experts (the Mixtral results)

def test_route_rows_layout():
    """Rows grouped by expert, tokens ascending inside an expert, every
    (token, expert) pair of the routing exactly once; offsets = histogram."""
    wl = workloads.make_moe(50, 128, 8, 6, topk=2, seed=3)
    ri, off = workloads.route_rows(wl.experts, 6)
    assert off[0] == 0 and off[-1] == 100
    assert np.array_equal(np.diff(off), np.bincount(wl.experts.reshape(-1), minlength=6))
    pairs = sorted((int(e), int(t)) for t in range(50) for e in wl.experts[t])
    got = [(e, int(ri[i])) for e in range(6) for i in range(off[e], off[e + 1])]
    assert got == pairs


def test_moe_single_expert_is_the_dense_layer():
    """E = 1 with every token routed to it: the dense Integer-Scale layer."""
    wl = workloads.make_linear(24, 512, 136, x_dtype="bf16", seed=11)
    ri, off = workloads.route_rows(np.zeros((24, 1), np.int64), 1)
    for alpha in (1024, None):
        moe = oracle.moe_intscale(wl.x, [wl.w], ri, off, alpha=alpha, out="f32")
        dense = oracle.linear_intscale(wl.x, wl.w, alpha=alpha, out="f32")
        assert moe["alpha"] == dense["alpha"]
        assert np.array_equal(moe["acc"], dense["acc"])
        assert np.array_equal(moe["y"], dense["y"])


def test_moe_identical_experts_repeat_the_dense_rows():
    """All experts equal: both routed rows of a token equal its dense row."""
    wl = workloads.make_linear(20, 256, 64, x_dtype="bf16", seed=12)
    route = np.array([[t % 3, (t + 1) % 3] for t in range(20)], np.int64)
    ri, off = workloads.route_rows(route, 3)
    moe = oracle.moe_intscale(wl.x, [wl.w] * 3, ri, off, alpha=1024, out="f32")
    dense = oracle.linear_intscale(wl.x, wl.w, alpha=1024, out="f32")
    assert np.array_equal(moe["acc"], dense["acc"][ri.astype(np.int64)])


def test_moe_shared_amplifier_postcondition():
    """One amplifier for the layer: the smallest power of two that lifts every
    positive group scale of every expert to at least 1."""
    wl = workloads.make_moe(8, 256, 32, 4, seed=5)
    wl.w[2] *= np.float32(0.05)  # one expert with much smaller scales sets the amplifier
    ri, off = workloads.route_rows(wl.experts, 4)
    moe = oracle.moe_intscale(wl.x, wl.w, ri, off, alpha=None)
    a = moe["alpha"]
    allpos = np.concatenate([sg[sg > 0].reshape(-1) for sg in moe["s_g"]]).astype(np.float64)
    assert (allpos * a >= 1.0).all()
    assert a == 1 or (allpos * (a // 2) < 1.0).any()
    assert a >= max(oracle.amplifier_search(sg) for sg in moe["s_g"])


def test_moe_rows_follow_their_token_and_expert():
    """Permuting the tokens moves rows, not values: the row of (token, expert)
    is a function of that pair only."""
    wl = workloads.make_moe(12, 256, 40, 3, seed=6)
    ri, off = workloads.route_rows(wl.experts, 3)
    base = oracle.moe_intscale(wl.x, wl.w, ri, off, alpha=1024)
    perm = np.random.default_rng(0).permutation(12)
    ri2, off2 = workloads.route_rows(wl.experts[perm], 3)
    other = oracle.moe_intscale(wl.x[perm], wl.w, ri2, off2, alpha=1024)
    assert np.array_equal(off, off2)
    for e in range(3):
        a = {int(t): base["acc"][i] for t, i in zip(ri[off[e]:off[e + 1]], range(off[e], off[e + 1]))}
        for i in range(off2[e], off2[e + 1]):
            assert np.array_equal(other["acc"][i], a[int(perm[ri2[i]])])


# ------------------------------------------------------------- amplifier analysis (Fig. 4)

def test_alpha_sweep_hand_case():
    # one group of two codes, s = 0.3: S = rne(0.3 alpha) = 0, 1, 1 for alpha = 1, 2, 4;
    # MSE = mean((q (S/alpha - 0.3))^2) = (49 + 9) d^2 / 2 with d = -0.3, 0.2, -0.05
    q = np.array([[7], [-3]], np.int8)
    s = np.array([[0.3]], np.float32)
    mse, bits = oracle.alpha_sweep(q, s, [1, 2, 4], group=2)
    np.testing.assert_allclose(mse, [2.61, 1.16, 0.0725], rtol=1e-6)
    assert bits.tolist() == [0, 1, 1]


def test_alpha_sweep_rounding_bound():
    # |S/alpha - s| <= 1/(2 alpha) per group, so MSE <= mean(q^2) / (4 alpha^2)
    rng = np.random.default_rng(21)
    w = (rng.standard_normal((512, 64)) * 0.02).astype(np.float32)
    q, s = oracle.quantize_groups(w, 128)
    alphas = [1 << j for j in range(15)]
    mse, bits = oracle.alpha_sweep(q, s, alphas, group=128)
    bound = np.mean(q.astype(np.float64) ** 2) / (4.0 * np.array(alphas, np.float64) ** 2)
    assert np.all(mse <= bound * (1 + 1e-12))
    assert np.all(np.diff(bits) >= 0) and bits[-1] > bits[0]


def test_alpha_sweep_exact_when_scales_are_multiples():
    # s_g = j / 1024 exactly: integer scales reproduce the float scales at alpha >= 1024
    q = np.array([[7, -5], [3, 2], [-7, 1], [0, -3]], np.int8)
    s = np.array([[37 / 1024, 5 / 1024]], np.float32)
    mse, _ = oracle.alpha_sweep(q, s, [256, 1024, 4096], group=4)
    assert mse[1] == 0.0 and mse[2] == 0.0 and mse[0] > 0.0


def test_alpha_sweep_bit_counts():
    # the largest S as an unsigned integer: 255 needs 8 bits, 256 needs 9
    q = np.ones((2, 2), np.int8)
    s = np.array([[255.0, 1.0]], np.float32)
    _, bits = oracle.alpha_sweep(q, s, [1], group=2)
    assert bits.tolist() == [8]
    s = np.array([[256.0, 3.0]], np.float32)
    _, bits = oracle.alpha_sweep(q, s, [1], group=2)
    assert bits.tolist() == [9]


# ------------------------------------------------------------- full int4 range [-8, 7]

def _nearest_code_brute(t, lo, hi):
    """Nearest integer code in [lo, hi] to t, ties to the even code."""
    codes = np.arange(lo, hi + 1, dtype=np.int64)
    d = np.abs(t[..., None].astype(np.float64) - codes)
    nearest = d == d.min(axis=-1, keepdims=True)
    nearest_even = nearest & (codes % 2 == 0)
    idx = np.where(nearest_even.any(axis=-1), nearest_even.argmax(axis=-1), nearest.argmax(axis=-1))
    return codes[idx]


def test_full_range_codes_brute_force():
    rng = np.random.default_rng(31)
    w = (rng.standard_normal((256, 40)) * 0.02).astype(np.float32)
    q, s = oracle.quantize_groups(w, 128, qmin=-8)
    sg = np.repeat(s, 128, axis=0)
    # the scale: one fp32 division of the group's max |w| by 8
    amax = np.abs(w).reshape(2, 128, 40).max(axis=1).astype(np.float32)
    assert np.array_equal(s, (amax / np.float32(8)).astype(np.float32))
    t = (w / sg).astype(np.float32)
    assert np.array_equal(q.astype(np.int64), _nearest_code_brute(t, -8, 7))
    assert q.min() >= -8 and q.max() <= 7


def test_full_range_extremes():
    # group 0's extreme is negative: it maps to -8 exactly; group 1's is positive: it clips to 7
    w = np.zeros((16, 1), np.float32)
    w[:8, 0] = [0.1, -0.8, 0.3, 0.05, -0.2, 0.7, 0.0, 0.35]
    w[8:, 0] = [0.8, -0.1, 0.3, 0.75, -0.7, 0.2, 0.0, -0.35]
    q, s = oracle.quantize_groups(w, 8, qmin=-8)
    assert s[0, 0] == np.float32(0.8) / np.float32(8) and s[1, 0] == np.float32(0.8) / np.float32(8)
    assert q[1, 0] == -8 and q[8, 0] == 7 and q[11, 0] == 7  # 0.75 / 0.1 = 7.5 rounds to 8, clips to 7
    err = np.abs(w[:, 0].astype(np.float64) - q[:, 0] * np.repeat(s[:, 0], 8).astype(np.float64))
    sg = np.repeat(s[:, 0], 8).astype(np.float64)
    inside = np.abs(w[:, 0] / np.repeat(s[:, 0], 8)) <= 7.5
    assert np.all(err[inside] <= sg[inside] / 2 * (1 + 1e-6))
    assert np.all(err[~inside] <= sg[~inside] * (1 + 1e-6))
    # the default range never uses -8
    q7, _ = oracle.quantize_groups(w, 8)
    assert q7.min() >= -7


# ------------------------------------------------------------- 8-bit weight codes (W8A8)

def test_groups_qmax127_brute_force():
    rng = np.random.default_rng(41)
    w = (rng.standard_normal((256, 24)) * 0.02).astype(np.float32)
    q, s = oracle.quantize_groups(w, 128, qmax=127)
    amax = np.abs(w).reshape(2, 128, 24).max(axis=1).astype(np.float32)
    assert np.array_equal(s, (amax / np.float32(127)).astype(np.float32))
    t = (w / np.repeat(s, 128, axis=0)).astype(np.float32)
    assert np.array_equal(q.astype(np.int64), _nearest_code_brute(t, -127, 127))
    # every group's extreme reaches +-127
    assert np.array_equal(np.abs(q).reshape(2, 128, 24).max(axis=1), np.full((2, 24), 127))


def test_linear_w8a8_layout_and_accumulators():
    rng = np.random.default_rng(42)
    x = rng.standard_normal((3, 256)).astype(np.float32)
    w = (rng.standard_normal((256, 16)) * 0.02).astype(np.float32)
    r = oracle.linear_intscale(x, w, group=128, alpha=4096, wbits=8, out="f32")
    assert r["packed"].shape == (16, 256) and r["packed"].dtype == np.int8
    assert np.array_equal(r["packed"], r["qw"].T)
    # the accumulators equal the dense int64 product with the integer weights W_int = S * q
    Wint = np.repeat(r["S"].astype(np.int64), 128, axis=0) * r["qw"].astype(np.int64)
    assert np.array_equal(r["acc"], r["qx"].astype(np.int64) @ Wint)


# ------------------------------------------------------------- asymmetric activations

def test_asym_golden_rows():
    g = _golden("quantize_int8_asymmetric.json")
    for case in g["cases"]:
        q, s, z = oracle.quantize_act_per_token_asym(np.array([case["x"]], np.float32))
        assert q[0].tolist() == case["q"], case["derivation"]
        assert _bits(s[0]) == int(case["s_bits"], 16), case["derivation"]
        assert int(z[0]) == case["z"], case["derivation"]


def _skewed_rows(rng, R, C, shift):
    x = rng.standard_normal((R, C)).astype(np.float32) + np.float32(shift)
    x[:, rng.choice(C, 3, replace=False)] *= np.float32(20)
    x[:, 0] = 0.0  # every row spans zero
    x[:, 1] = -abs(x[:, 1]) - 0.1
    return x


def test_asym_codes_are_the_nearest_grid_points():
    """Each code is the nearest integer of x/s + z in [-128, 127] (ties to
    even), searched by brute force; the scale is the range over 255 to within
    the one fp32 rounding of each step, and z is within 1/2 of the real-valued
    zero point -128 - x_min / s."""
    rng = np.random.default_rng(51)
    x = _skewed_rows(rng, 12, 384, 1.5)
    q, s, z = oracle.quantize_act_per_token_asym(x)
    lo = x.min(axis=1).astype(np.float64)
    hi = x.max(axis=1).astype(np.float64)
    assert np.all(np.abs(s - (hi - lo) / 255) <= 2 * np.spacing(s))
    zr = -128 - lo / s.astype(np.float64)
    assert np.all(np.abs(z - zr) <= 0.5 + 1e-4)
    t = (x / s[:, None]).astype(np.float32).astype(np.float64) + z[:, None]
    assert np.array_equal(q.astype(np.int64), _nearest_code_brute(t, -128, 127))


def test_asym_zero_exact_extremes_and_error_bound():
    rng = np.random.default_rng(52)
    x = _skewed_rows(rng, 16, 256, 2.0)
    q, s, z = oracle.quantize_act_per_token_asym(x)
    # zero is exactly representable: x = 0 gets code z, x_hat = 0
    assert np.array_equal(q[:, 0].astype(np.int64), z.astype(np.int64))
    # the range ends land on the extreme codes (to within one rounding step)
    rows = np.arange(x.shape[0])
    assert np.all(q[rows, x.argmin(axis=1)] <= -127)
    assert np.all(q[rows, x.argmax(axis=1)] >= 126)
    # every value lies in the grid's range, so |x - s (q - z)| <= s/2
    xh = s[:, None].astype(np.float64) * (q.astype(np.float64) - z[:, None])
    err = np.abs(x - xh)
    assert np.all(err <= s[:, None] * (0.5 + 1e-4))
    # round-to-nearest error has variance about s^2 / 12
    var = np.mean((err / s[:, None]) ** 2)
    assert abs(var - 1 / 12) < 0.01


def test_asym_constant_rows_and_scale_zero():
    x = np.array([[3.0] * 8, [-0.75] * 8, [0.0] * 8], np.float32)
    q, s, z = oracle.quantize_act_per_token_asym(x)
    xh = s[:, None].astype(np.float64) * (q.astype(np.float64) - z[:, None])
    assert np.allclose(xh[:2], x[:2], rtol=1e-6)
    assert s[2] == 0 and z[2] == 0 and not q[2].any()


def test_asym_beats_symmetric_on_one_sided_rows():
    """The notes recommend asymmetric codes for activations that are not
    centred on zero: on a shifted distribution its reconstruction error is
    smaller than the symmetric one's."""
    rng = np.random.default_rng(53)
    x = np.abs(rng.standard_normal((8, 512))).astype(np.float32)
    x[:, 0] = 0.0
    qa, sa, za = oracle.quantize_act_per_token_asym(x)
    qs, ss = oracle.quantize_act_per_token(x)
    ea = np.mean((x - sa[:, None] * (qa.astype(np.float64) - za[:, None])) ** 2)
    es = np.mean((x - ss[:, None] * qs.astype(np.float64)) ** 2)
    assert ea < 0.5 * es


def test_intscale_acc_asym_reduces_to_symmetric_when_z_is_zero():
    rng = np.random.default_rng(54)
    qx = rng.integers(-128, 128, (3, 256)).astype(np.int8)
    qw = rng.integers(-7, 8, (256, 10)).astype(np.int8)
    S = rng.integers(1, 300, (2, 10)).astype(np.int32)
    assert np.array_equal(oracle.intscale_acc_asym(qx, np.zeros(3, np.int32), qw, S),
                          oracle.intscale_acc(qx, qw, S))


def test_intscale_acc_asym_equals_the_expanded_zero_point_form():
    """(q_X - Z_X) q_W expands to q_W q_X - Z_X q_W: the second term is z[m]
    times the column sum of the integer weights S * q_W, precomputable per
    column; checked with numpy int64 matmuls."""
    rng = np.random.default_rng(55)
    M, K, N = 5, 384, 12
    qx = rng.integers(-128, 128, (M, K)).astype(np.int8)
    z = rng.integers(-128, 128, M).astype(np.int32)
    qw = rng.integers(-8, 8, (K, N)).astype(np.int8)
    S = rng.integers(1, 2000, (K // 128, N)).astype(np.int32)
    Wint = np.repeat(S.astype(np.int64), 128, axis=0) * qw.astype(np.int64)
    expanded = qx.astype(np.int64) @ Wint - z.astype(np.int64)[:, None] * Wint.sum(axis=0)[None, :]
    assert np.array_equal(oracle.intscale_acc_asym(qx, z, qw, S), expanded)


def test_linear_asym_bruteforce_dequantized_fp64():
    """acc * s_a / alpha equals the fp64 matmul of the dequantized operands
    s_a (q_x - z) and S / alpha q_w on tiny inputs."""
    rng = np.random.default_rng(56)
    for _ in range(150):
        M = int(rng.integers(1, 5))
        N = int(rng.integers(1, 9))
        K = int(rng.choice([128, 256]))
        x = (rng.standard_normal((M, K)) + rng.uniform(-2, 2)).astype(np.float32)
        w = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
        alpha = int(rng.choice([1024, 256]))
        r = oracle.linear_intscale(x, w, alpha=alpha, out="f32", asym=True)
        xh = r["s_a"][:, None].astype(np.float64) * (r["qx"].astype(np.float64) - r["z"][:, None])
        wh = np.repeat(r["S"], 128, axis=0).astype(np.float64) / alpha * r["qw"]
        ref = xh @ wh
        assert np.allclose(r["y64"], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
        # on rows that span zero the activation side is within half a step of x
        span = (x.min(axis=1) < 0) & (x.max(axis=1) > 0)
        assert np.all(np.abs(x - xh)[span] <= (r["s_a"][:, None] * (0.5 + 1e-4) + 0 * xh)[span])


def test_asym_error_analysis_trend():
    """The oracle-side analysis (oracle/asym_error.py) on a small layer: while
    the rows span zero (offsets up to 2 here), the asymmetric codes' error is
    below the symmetric one's and the gap grows with the offset.  Further off
    zero a row's range excludes zero, the printed clip of z acts and the
    asymmetric codes lose the row's far end (the notes' formulas as printed)."""
    from oracle import asym_error

    rows = {r["offset"]: r for r in asym_error.analyse(M=8, K=512, N=64, outliers=False)}
    for off in (0.0, 0.5, 1.0, 2.0):
        assert rows[off]["act_mse_asym"] < rows[off]["act_mse_sym"]
        assert rows[off]["out_rel_rms_err_act_only_asym"] < rows[off]["out_rel_rms_err_act_only_sym"]
    gap = [rows[o]["out_rel_rms_err_act_only_sym"] - rows[o]["out_rel_rms_err_act_only_asym"] for o in (0.5, 1.0, 2.0)]
    assert gap[0] < gap[1] < gap[2]
    assert rows[4.0]["act_mse_asym"] > rows[4.0]["act_mse_sym"]
