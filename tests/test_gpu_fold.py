"""Integer scales folded into the unpacked weight operand.

A CTA of the tile kernel (128-token tiles) whose integer scales all lie in
[0, 16] (or in [0, 18] for groups without the code -8) writes S * q as the
MMA operand (then in int8) and accumulates the whole segment in TMEM; any
other CTA drains each group and multiplies by S.  The sum is the same integer either way, so every case
here is bit-exact against the oracle's accumulators.

The weights are built so that quantizing them gives chosen codes and scales
exactly: w[k,n] = q[k,n] * S[g,n] / 1024 with a code of largest magnitude in
every (group, column), so that max|w| / qmax = S / 1024 and the integer scale
at alpha = 1024 is S.  This reaches the edges of the folded range (S = 16
with the code -8 gives the operand byte -128; S = 0 gives zero groups)."""
import numpy as np
import pytest
import torch

import bit_gemm_quantize_b200 as bgq
import oracle
from bit_gemm_quantize_b200 import workloads

pytestmark = pytest.mark.gpu

ALPHA = 1024


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _weights(K, N, group, rng, full_range, s_hi=16, band=None, band_hi=200):
    """w [K, N] fp32 whose group quantization gives codes q and scales S
    (S in [0, s_hi]; columns in `band` up to band_hi)."""
    G = K // group
    S = rng.integers(0, s_hi + 1, size=(G, N))
    S[rng.random((G, N)) < 0.25] = s_hi  # the edge value often
    if band is not None:
        S[:, band[0]:band[1]] = rng.integers(17, band_hi + 1, size=(G, band[1] - band[0]))
    lo = -8 if full_range else -7
    q = rng.integers(lo, 8, size=(K, N))
    ext = -8 if full_range else 7
    q[::group, :] = ext  # every (group, column) reaches the code of largest magnitude
    q[np.repeat(S, group, axis=0) == 0] = 0  # a zero scale quantizes its group to zero codes
    w = q.astype(np.float64) * np.repeat(S, group, axis=0).astype(np.float64) / ALPHA
    return w.astype(np.float32), q.astype(np.int8), S.astype(np.int32)


def _tokens(M, K, rng):
    qx = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    qx[:, ::97] = -127
    s_a = (rng.random(M) * 0.05 + 1e-3).astype(np.float32)
    return qx, s_a


def _check(M, K, N, group, full_range, seed, **kw):
    dev = _dev()
    rng = np.random.default_rng(seed)
    w, q, S = _weights(K, N, group, rng, full_range, **kw)
    qx, s_a = _tokens(M, K, rng)
    qmin = -8 if full_range else -7
    pk = bgq.pack_w4_groupwise(torch.from_numpy(w).to(dev), group=group, alpha=ALPHA, qmin=qmin)
    # the packing recovers the chosen codes and scales (oracle side)
    qw, sg = oracle.quantize_groups(w, group, qmin=-8 if full_range else None)
    assert np.array_equal(qw, q)
    assert np.array_equal(oracle.integer_scales(sg, ALPHA), S)
    assert np.array_equal(pk["S"].cpu().numpy().astype(np.int32), S)
    q_d = torch.from_numpy(qx).to(dev)
    s_d = torch.from_numpy(s_a).to(dev)
    acc = bgq.w4a8_gemm_intscale(q_d, s_d, pk["packed"], pk["S"], ALPHA, group=group, out="i32")
    ref = oracle.intscale_acc(qx, q, S, group)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref)
    y = bgq.w4a8_gemm_intscale(q_d, s_d, pk["packed"], pk["S"], ALPHA, group=group, out="f32").cpu().numpy()
    y_ref = ref.astype(np.float64) * s_a[:, None].astype(np.float64) / ALPHA
    tau = max(1e-2 * np.sqrt(np.mean(np.square(y_ref))), 1e-30)
    assert (np.abs(y - y_ref) / np.maximum(np.abs(y_ref), tau)).max(initial=0.0) <= 1e-5
    assert bgq.device_status() == 0


# token tiles 16 (two CTAs per SM), 32 and 64 (these always drain) and 128;
# ragged N; groups of one and of two K blocks; split tiles
FOLD_CASES = [
    (8, 1024, 520, 128),
    (24, 2048, 264, 256),
    (64, 512, 1032, 128),
    (300, 1024, 392, 128),
    (1024, 4096, 1024, 128),
]


@pytest.mark.parametrize("full_range", [True, False])
@pytest.mark.parametrize("M,K,N,group", FOLD_CASES)
def test_folded_scales_bitexact(M, K, N, group, full_range):
    _check(M, K, N, group, full_range, seed=M + K + N + int(full_range))


@pytest.mark.parametrize("M,K,N,group", [(8, 1024, 1032, 128), (300, 2048, 776, 256), (1024, 4096, 1024, 128)])
def test_folded_and_drained_ctas_mixed(M, K, N, group):
    """Columns 256..383 carry scales of 17 to 200 in groups that all hold the
    code -8: the CTAs that meet them drain every group, the others fold;
    tiles split between the two kinds combine."""
    _check(M, K, N, group, True, seed=5 * M + N, band=(256, 384))


@pytest.mark.parametrize("M,K,N", [(130, 1024, 520), (512, 2048, 1024)])
@pytest.mark.parametrize("big", [17, 18, 40, 200])
def test_a_few_scales_above_16(M, K, N, big):
    """A few groups with one scale above 16 and codes in [-7, 7]: scales of
    17 and 18 still fold (S * q stays in int8 without the code -8); the CTAs
    that meet a larger one drain, the others fold."""
    dev = _dev()
    rng = np.random.default_rng(big + M)
    group = 128
    w, q, S = _weights(K, N, group, rng, False)
    for g, n in [(3, 200), (0, N - 1), (K // group - 1, 7), (1, N // 2)]:
        S[g, n] = big
        q[g * group, n] = 7  # the group's largest code (its codes may have been zeroed with a zero scale)
        w[g * group:(g + 1) * group, n] = (q[g * group:(g + 1) * group, n].astype(np.float64) * big /
                                           ALPHA).astype(np.float32)
    qx, s_a = _tokens(M, K, rng)
    pk = bgq.pack_w4_groupwise(torch.from_numpy(w).to(dev), group=group, alpha=ALPHA)
    assert np.array_equal(pk["S"].cpu().numpy().astype(np.int32), S)
    acc = bgq.w4a8_gemm_intscale(torch.from_numpy(qx).to(dev), torch.from_numpy(s_a).to(dev), pk["packed"],
                                 pk["S"], ALPHA, group=group, out="i32")
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), oracle.intscale_acc(qx, q, S, group))
    assert bgq.device_status() == 0


@pytest.mark.parametrize("routed", [True, False])
def test_grouped_experts_fold_and_drain(routed):
    """The grouped expert call: expert 0's scales fold, expert 1's do not
    (scales up to 120), expert 2 has both kinds of columns."""
    dev = _dev()
    rng = np.random.default_rng(23)
    T, K, N, E, group = 300, 1024, 392, 3, 128
    ws = [_weights(K, N, group, rng, False)[0],
          _weights(K, N, group, rng, False, band=(0, N), band_hi=120)[0],
          _weights(K, N, group, rng, False, band=(128, 256), band_hi=60)[0]]
    x = rng.standard_normal((T, K)).astype(np.float32)
    experts = np.stack([rng.permutation(E)[:2] for _ in range(T)])
    ri, off = workloads.route_rows(experts, E)
    ri_d = torch.from_numpy(ri.astype(np.int32)).to(dev)
    off_d = torch.from_numpy(np.asarray(off, np.int64)).to(dev)
    xd = torch.from_numpy(x).to(dev)
    pk = bgq.pack_moe_experts([torch.from_numpy(w).to(dev) for w in ws], alpha=ALPHA)
    assert pk["alpha"] == ALPHA
    if routed:
        q, s = bgq.quantize_act_routed(xd, ri_d)
        rows = None
    else:
        q, s = bgq.quantize_act_per_token(xd)
        rows = ri_d
    acc = bgq.w4a8_gemm_intscale_grouped(q, s, rows, off_d, pk["packed"], pk["S"], ALPHA, out="i32")
    ref = oracle.moe_intscale(x, ws, ri, off, alpha=ALPHA)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref["acc"])
    assert bgq.device_status() == 0
