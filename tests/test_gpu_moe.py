"""Mixture-of-experts path on the GPU against the oracle: one grouped call
(device routing offsets and pointer arrays) runs every expert's integer-scale
GEMM over its routed rows with a shared amplifier (the Integer Scale summary's
Mixtral results)."""
import numpy as np
import pytest
import torch

import bit_gemm_quantize_b200 as bgq
import oracle
from bit_gemm_quantize_b200 import workloads

pytestmark = pytest.mark.gpu


def _close(y, y_ref, out):
    ref = np.asarray(y_ref, np.float64)
    tau = 1e-2 * np.sqrt(np.mean(ref * ref)) if ref.size else 0.0
    rtol = 1e-3 if out == "f32" else 4e-3
    err = np.abs(np.asarray(y, np.float64) - ref)
    assert np.all(err <= rtol * np.maximum(np.abs(ref), tau))


def _grouped(q, s, ri, off, pk, alpha, out, **kw):
    dev = q.device
    return bgq.w4a8_gemm_intscale_grouped(q, s, torch.from_numpy(np.asarray(ri, np.int32)).to(dev),
                                          torch.from_numpy(np.asarray(off, np.int64)).to(dev), pk["packed"], pk["S"],
                                          alpha, out=out, **kw)


def _run(wl, E, alpha, out="i32", route=None, routed=False):
    """routed: quantize the tokens in routed order and hand the grouped call
    those rows with no row index (whole-tile reads); otherwise quantize every
    token once and let the call gather rows by index."""
    dev = torch.device("cuda:0")
    route = wl.experts if route is None else route
    ri, off = workloads.route_rows(route, E)
    x = torch.from_numpy(wl.x).to(dev).to(torch.bfloat16)
    pk = bgq.pack_moe_experts([torch.from_numpy(w).to(dev) for w in wl.w], alpha=alpha)
    if routed:
        q, s = bgq.quantize_act_routed(x, torch.from_numpy(ri.astype(np.int32)).to(dev))
        y = bgq.w4a8_gemm_intscale_grouped(q, s, None, torch.from_numpy(np.asarray(off, np.int64)).to(dev),
                                           pk["packed"], pk["S"], pk["alpha"], out=out)
    else:
        q, s = bgq.quantize_act_per_token(x)
        y = _grouped(q, s, ri, off, pk, pk["alpha"], out)
    torch.cuda.synchronize()
    return ri, off, pk, y


@pytest.mark.parametrize("T,K,N,E,topk", [(64, 512, 256, 4, 2), (37, 256, 136, 8, 2), (200, 1024, 520, 3, 1),
                                          (700, 512, 384, 2, 1)])
@pytest.mark.parametrize("alpha", [1024, None])
@pytest.mark.parametrize("routed", [False, True])
def test_moe_parity(T, K, N, E, topk, alpha, routed):
    wl = workloads.make_moe(T, K, N, E, topk=topk, seed=T + E)
    ri, off, pk, acc = _run(wl, E, alpha, "i32", routed=routed)
    ref = oracle.moe_intscale(wl.x, wl.w, ri, off, alpha=alpha, out="f32")
    assert pk["alpha"] == ref["alpha"]
    for e in range(E):
        assert np.array_equal(pk["packed"][e].cpu().numpy(), ref["packed"][e])
        assert np.array_equal(pk["S"][e].cpu().numpy(), ref["S"][e])
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref["acc"])
    for out in ("f32", "f16"):
        _, _, _, y = _run(wl, E, alpha, out, routed=routed)
        _close(y.float().cpu().numpy(), ref["y64"], out)
    assert bgq.device_status() == 0


@pytest.mark.parametrize("T,K,x_dtype", [(50, 4096, "bf16"), (33, 16384, "f32"), (5, 256, "f32")])
def test_routed_quantize_matches_per_token_codes(T, K, x_dtype):
    """Row i of the routed quantization is token row_index[i]'s codes and
    scale, bit for bit (the oracle's per-token quantization, gathered);
    tokens repeat, skip and come in any order."""
    dev = torch.device("cuda:0")
    wl = workloads.make_linear(T, K, 8, x_dtype=x_dtype, seed=T)
    qx, s_a = oracle.quantize_act_per_token(wl.x)
    rng = np.random.default_rng(T)
    ri = rng.integers(0, T, 3 * T).astype(np.int32)
    x = torch.from_numpy(wl.x).to(dev)
    if x_dtype == "bf16":
        x = x.to(torch.bfloat16)
    q, s = bgq.quantize_act_routed(x, torch.from_numpy(ri).to(dev))
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), qx[ri])
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_a[ri].view(np.uint32))
    assert bgq.device_status() == 0


def test_routed_quantize_out_of_range_token():
    """A routed row naming a token outside [0, T) gets zero codes and scale,
    and the device status word reports W4A8_ERR_INVALID_ARG (1)."""
    dev = torch.device("cuda:0")
    wl = workloads.make_linear(8, 512, 8, x_dtype="f32", seed=3)
    qx, s_a = oracle.quantize_act_per_token(wl.x)
    ri = np.array([2, -1, 7, 8, 0], np.int32)
    bgq.device_status(clear=True)
    q, s = bgq.quantize_act_routed(torch.from_numpy(wl.x).to(dev), torch.from_numpy(ri).to(dev))
    torch.cuda.synchronize()
    assert bgq.device_status(clear=True) == 1
    qh, sh = q.cpu().numpy(), s.cpu().numpy()
    for i, t in enumerate(ri):
        if 0 <= t < 8:
            assert np.array_equal(qh[i], qx[t]) and sh[i] == s_a[t]
        else:
            assert not qh[i].any() and sh[i] == 0.0


def test_moe_empty_experts_and_single_expert():
    wl = workloads.make_moe(48, 512, 256, 5, topk=1, seed=9)
    route = np.full((48, 1), 3, np.int64)  # every token to expert 3, experts 0, 1, 2, 4 empty
    ri, off, pk, acc = _run(wl, 5, 1024, "i32", route)
    ref = oracle.moe_intscale(wl.x, wl.w, ri, off, alpha=1024)
    assert list(np.diff(off)) == [0, 0, 0, 48, 0]
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref["acc"])
    _, _, _, acc_r = _run(wl, 5, 1024, "i32", route, routed=True)
    assert np.array_equal(acc_r.cpu().numpy().astype(np.int64), ref["acc"])
    # no routed rows at all: nothing to do
    dev = torch.device("cuda:0")
    q = torch.zeros((4, 512), dtype=torch.int8, device=dev)
    s = torch.ones((4,), dtype=torch.float32, device=dev)
    y = bgq.w4a8_gemm_intscale_grouped(q, s, torch.zeros((0,), dtype=torch.int32, device=dev),
                                       torch.zeros((3,), dtype=torch.int64, device=dev), [None, None], [None, None],
                                       1024, N=256)
    assert y.shape == (0, 256)


def test_moe_output_rows_in_token_slot_order():
    """out_row = token * top_k + slot returns every token's top-k outputs
    side by side ([T, top_k, N]) with no gather or permute afterwards."""
    T, K, N, E, topk = 150, 512, 256, 5, 2
    wl = workloads.make_moe(T, K, N, E, topk=topk, seed=12)
    ri, off = workloads.route_rows(wl.experts, E)
    # the slot of each routed row: position of its expert in the token's routing
    exp_of_row = np.repeat(np.arange(E), np.diff(off))
    slot = np.array([int(np.nonzero(wl.experts[t] == e)[0][0]) for t, e in zip(ri, exp_of_row)])
    out_row = (ri.astype(np.int64) * topk + slot).astype(np.int32)
    dev = torch.device("cuda:0")
    q, s = bgq.quantize_act_per_token(torch.from_numpy(wl.x).to(dev).to(torch.bfloat16))
    pk = bgq.pack_moe_experts([torch.from_numpy(w).to(dev) for w in wl.w], alpha=1024)
    y = _grouped(q, s, ri, off, pk, 1024, "i32", out_row=torch.from_numpy(out_row).to(dev), y_rows=T * topk)
    torch.cuda.synchronize()
    ref = oracle.moe_intscale(wl.x, wl.w, ri, off, alpha=1024)
    want = np.zeros((T * topk, N), np.int64)
    want[out_row] = ref["acc"]
    assert np.array_equal(y.cpu().numpy().astype(np.int64), want)
    assert bgq.device_status() == 0


def test_moe_out_of_range_token_index_is_reported():
    """A routed row naming a token outside [0, T) is written as zeros and the
    device status word reports W4A8_ERR_INVALID_ARG (1); the other rows are right."""
    dev = torch.device("cuda:0")
    wl = workloads.make_moe(16, 256, 128, 2, topk=1, seed=4)
    ri, off = workloads.route_rows(wl.experts, 2)
    ri_bad = ri.copy()
    ri_bad[0] = 1000
    x = torch.from_numpy(wl.x).to(dev).to(torch.bfloat16)
    q, s = bgq.quantize_act_per_token(x)
    pk = bgq.pack_moe_experts([torch.from_numpy(w).to(dev) for w in wl.w], alpha=1024)
    bgq.device_status(clear=True)
    acc = _grouped(q, s, ri_bad, off, pk, 1024, "i32")
    torch.cuda.synchronize()
    assert bgq.device_status(clear=True) == 1
    ref = oracle.moe_intscale(wl.x, wl.w, ri, off, alpha=1024)
    a = acc.cpu().numpy().astype(np.int64)
    assert np.all(a[0] == 0)
    assert np.array_equal(a[1:], ref["acc"][1:])


def test_moe_mixtral_shaped_sampled():
    """A Mixtral-shaped layer slice (K = 4096, 8 experts, top-2, 256 tokens,
    N = 2048): raw accumulators at sampled (row, column) positions."""
    T, K, N, E = 256, 4096, 2048, 8
    wl = workloads.make_moe(T, K, N, E, topk=2, seed=21)
    ri, off, pk, acc = _run(wl, E, None, "i32")
    qx, s_a = oracle.quantize_act_per_token(wl.x)
    rng = np.random.default_rng(5)
    a = acc.cpu().numpy().astype(np.int64)
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        qw, sg = oracle.quantize_groups(wl.w[e], 128)
        S = oracle.integer_scales(sg, pk["alpha"])
        ms = rng.integers(0, hi - lo, 40)
        ns = rng.integers(0, N, 40)
        want = oracle.intscale_acc_at(qx[ri[lo:hi].astype(np.int64)], qw, S, ms, ns)
        assert np.array_equal(a[lo + ms, ns], want)


def test_moe_mixtral_full_layer_sampled():
    """The whole Mixtral-shaped layer the benchmark times: 2048 tokens, 8
    experts of W [4096, 14336], top-2 routing, one amplifier searched over all
    experts' group scales.  Codes, token scales, the amplifier and every
    expert's packed weights and integer scales bit-exact in full; raw
    accumulators and fp16 outputs at samples spread over every expert and
    every 128-column tile."""
    T, K, N, E = 2048, 4096, 14336, 8
    wl = workloads.make_moe(T, K, N, E, topk=2, seed=21)
    ri, off = workloads.route_rows(wl.experts, E)
    dev = torch.device("cuda:0")
    x = torch.from_numpy(wl.x).to(dev).to(torch.bfloat16)
    q, s = bgq.quantize_act_per_token(x)
    pk = bgq.pack_moe_experts([torch.from_numpy(w).to(dev) for w in wl.w], alpha=None)
    acc = _grouped(q, s, ri, off, pk, pk["alpha"], "i32")
    y = _grouped(q, s, ri, off, pk, pk["alpha"], "f16")
    # the routed rows quantized in routed order, read as whole tiles
    ri_d = torch.from_numpy(ri.astype(np.int32)).to(dev)
    q_r, s_r = bgq.quantize_act_routed(x, ri_d)
    acc_r = bgq.w4a8_gemm_intscale_grouped(q_r, s_r, None, torch.from_numpy(np.asarray(off, np.int64)).to(dev),
                                           pk["packed"], pk["S"], pk["alpha"], out="i32")
    torch.cuda.synchronize()
    assert bgq.device_status() == 0
    assert torch.equal(acc_r, acc)

    qx, s_a = oracle.quantize_act_per_token(wl.x)
    assert np.array_equal(q.cpu().numpy(), qx)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_a.view(np.uint32))
    qws, sgs = zip(*[oracle.quantize_groups(w, 128) for w in wl.w])
    alpha = oracle.amplifier_search(np.concatenate([sg.reshape(-1) for sg in sgs]))
    assert pk["alpha"] == alpha
    a = acc.cpu().numpy().astype(np.int64)
    yh = y.float().cpu().numpy()
    rng = np.random.default_rng(17)
    for e in range(E):
        S = oracle.integer_scales(sgs[e], alpha)
        oracle.check_worst_case(S, 128)
        assert np.array_equal(pk["S"][e].cpu().numpy().astype(np.int32), S)
        assert np.array_equal(pk["packed"][e].cpu().numpy(), oracle.pack_int4(qws[e]))
        lo, hi = int(off[e]), int(off[e + 1])
        assert hi > lo
        tiles = np.repeat(np.arange(N // 128), 2)  # two samples in every column tile
        ns = tiles * 128 + rng.integers(0, 128, tiles.size)
        ms = rng.integers(0, hi - lo, tiles.size)
        ms[:2] = [0, hi - lo - 1]  # the expert's first and last rows
        toks = ri[lo:hi].astype(np.int64)
        want = oracle.intscale_acc_at(qx[toks], qws[e], S, ms, ns)
        assert np.array_equal(a[lo + ms, ns], want)
        y_ref = want.astype(np.float64) * s_a[toks[ms]].astype(np.float64) / alpha
        _close(yh[lo + ms, ns], y_ref, "f16")
