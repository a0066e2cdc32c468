"""The C-ABI library: it loads, exports every function the header declares,
and rejects bad arguments on the host before touching the GPU (no compute
calls, so this runs without a GPU)."""
import ctypes
import os

import pytest

from bit_gemm_quantize_b200 import _native

OK, INVALID, SHAPE, ALIGN, DTYPE = 0, 1, 2, 3, 4
A = 0x10000  # a fake, 16-byte aligned "device" address: every call below fails its host-side
# checks (or is an M = 0 no-op) before any launch, so it is never dereferenced
U = 0x10001  # misaligned


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_native.LIB_PATH):
        from bit_gemm_quantize_b200 import build

        build.build()
    return _native.load()


def test_exports_every_declared_symbol(lib):
    names = _native.declared_symbols()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code in range(10):
        assert lib.w4a8_status_string(code) not in (None, b"", b"unknown status")
    assert lib.w4a8_status_string(99) == b"unknown status"


def _q(lib, x=A, dt=_native.BF16, M=4, K=256, ldx=256, q=A, s=A):
    return lib.quantize_act_per_token(ctypes.c_void_p(x), dt, M, K, ldx, ctypes.c_void_p(q), ctypes.c_void_p(s),
                                      None)


def test_quantize_argument_checks(lib):
    assert _q(lib, dt=_native.F16) == DTYPE
    assert _q(lib, dt=_native.I32) == DTYPE
    assert _q(lib, K=100) == SHAPE
    assert _q(lib, K=0) == SHAPE
    assert _q(lib, M=-1) == SHAPE
    assert _q(lib, ldx=128) == SHAPE
    assert _q(lib, M=0) == OK  # empty input is a no-op, nothing launched
    assert _q(lib, x=0) == INVALID
    assert _q(lib, s=0) == INVALID
    assert _q(lib, x=U) == ALIGN
    assert _q(lib, q=U) == ALIGN
    assert _q(lib, ldx=260) == ALIGN  # bf16 rows 520 bytes apart: not 16-byte aligned
    assert _q(lib, s=A + 2) == ALIGN  # fp32 scales: 4-byte aligned


def _is(lib, qx=A, sa=A, wp=A, S=A, alpha=1024, M=16, N=128, K=256, group=128, y=A, dt=_native.F16, ws=0, wsb=0):
    return lib.w4a8_gemm_intscale(ctypes.c_void_p(qx), ctypes.c_void_p(sa), ctypes.c_void_p(wp), ctypes.c_void_p(S),
                                  alpha, M, N, K, group, ctypes.c_void_p(y), dt, ctypes.c_void_p(ws), wsb, None)


def test_intscale_argument_checks(lib):
    assert _is(lib, K=200) == SHAPE
    assert _is(lib, group=64) == SHAPE
    assert _is(lib, K=384, group=256) == SHAPE
    assert _is(lib, N=100) == SHAPE
    assert _is(lib, N=0) == SHAPE
    assert _is(lib, M=-3) == SHAPE
    assert _is(lib, dt=_native.BF16) == DTYPE
    assert _is(lib, alpha=1000) == INVALID
    assert _is(lib, alpha=0) == INVALID
    assert _is(lib, alpha=-4) == INVALID
    assert _is(lib, M=0) == OK
    assert _is(lib, S=0) == INVALID
    assert _is(lib, y=0) == INVALID
    assert _is(lib, qx=U) == ALIGN
    assert _is(lib, wp=U) == ALIGN


def test_floatscale_argument_checks(lib):
    def fs(**kw):
        a = dict(qx=A, sa=A, wp=A, sg=A, M=16, N=128, K=256, group=128, y=A, dt=_native.F16)
        a.update(kw)
        return lib.w4a8_gemm_floatscale(ctypes.c_void_p(a["qx"]), ctypes.c_void_p(a["sa"]), ctypes.c_void_p(a["wp"]),
                                        ctypes.c_void_p(a["sg"]), a["M"], a["N"], a["K"], a["group"],
                                        ctypes.c_void_p(a["y"]), a["dt"], None, 0, None)

    assert fs(dt=_native.I32) == DTYPE  # raw accumulators exist only for integer scales
    assert fs(sg=0) == INVALID
    assert fs(K=130) == SHAPE
    assert fs(M=0) == OK


def test_pack_argument_checks(lib):
    def pk(w=A, K=256, N=128, group=128, alpha=1024, wp=A, sg=A, S=A, ws=A):
        a_out = ctypes.c_int32(0)
        c_out = ctypes.c_int64(0)
        return lib.pack_w4_groupwise(ctypes.c_void_p(w), K, N, group, alpha, ctypes.c_void_p(wp), ctypes.c_void_p(sg),
                                     ctypes.c_void_p(S), ctypes.byref(a_out), ctypes.byref(c_out), ctypes.c_void_p(ws),
                                     None)

    assert pk(K=200) == SHAPE
    assert pk(group=48) == SHAPE
    assert pk(N=12) == SHAPE
    assert pk(alpha=3) == INVALID
    assert pk(alpha=-1) == INVALID
    assert pk(w=0) == INVALID
    assert pk(sg=0) == INVALID
    assert pk(S=0) == INVALID  # packed given without integer scales
    assert pk(ws=0) == INVALID
    assert pk(w=U) == ALIGN


def test_workspace_size_without_device(lib):
    # M = 0 needs nothing; otherwise the size depends on the device's SM count
    assert lib.w4a8_gemm_workspace_size(0, 128, 256, 128, 0) == 0
    assert lib.w4a8_gemm_workspace_size(4, 100, 256, 128, 0) == 0  # invalid shape
    import torch

    if not torch.cuda.is_available():
        assert lib.w4a8_gemm_workspace_size(4, 128, 256, 128, 0) == -1


def test_binding_refuses_cpu_tensors():
    import torch

    x = torch.zeros(4, 256)
    with pytest.raises(ValueError):
        _native.quantize_act_per_token(x)
    with pytest.raises(ValueError):
        _native.pack_w4_groupwise(torch.zeros(256, 128))


def test_binding_fails_loudly_without_library(tmp_path):
    with pytest.raises(RuntimeError):
        saved = _native._lib
        _native._lib = None
        try:
            _native.load(str(tmp_path / "missing.so"))
        finally:
            _native._lib = saved


def test_range_and_w8_pack_argument_checks(lib):
    a_out = ctypes.c_int32(0)
    c_out = ctypes.c_int64(0)

    def pr(qmin=-8, K=256, group=128):
        return lib.pack_w4_groupwise_range(ctypes.c_void_p(A), K, 128, group, 1024, qmin, ctypes.c_void_p(A),
                                           ctypes.c_void_p(A), ctypes.c_void_p(A), ctypes.byref(a_out),
                                           ctypes.byref(c_out), ctypes.c_void_p(A), None)

    assert pr(qmin=-6) == INVALID
    assert pr(qmin=-9) == INVALID
    assert pr(K=200) == SHAPE

    def p8(w8=A, K=256, group=128, alpha=0):
        return lib.pack_w8_groupwise(ctypes.c_void_p(A), K, 128, group, alpha, ctypes.c_void_p(w8), ctypes.c_void_p(A),
                                     ctypes.c_void_p(A), ctypes.byref(a_out), ctypes.byref(c_out), ctypes.c_void_p(A),
                                     None)

    assert p8(K=200) == SHAPE
    assert p8(group=48) == SHAPE
    assert p8(w8=0) == INVALID
    assert p8(alpha=6) == INVALID
    assert p8(w8=U) == ALIGN

    def g8(M=16, K=256, dt=_native.F16, S=A):
        return lib.w8a8_gemm_intscale(ctypes.c_void_p(A), ctypes.c_void_p(A), ctypes.c_void_p(A), ctypes.c_void_p(S),
                                      1024, M, 128, K, 128, ctypes.c_void_p(A), dt, None, 0, None)

    assert g8(K=200) == SHAPE
    assert g8(dt=_native.BF16) == DTYPE
    assert g8(S=0) == INVALID
    assert g8(M=0) == OK


def test_asymmetric_argument_checks(lib):
    def qa(x=A, dt=_native.BF16, K=256, z=A):
        return lib.quantize_act_per_token_asym(ctypes.c_void_p(x), dt, 4, K, K, ctypes.c_void_p(A),
                                               ctypes.c_void_p(A), ctypes.c_void_p(z), None)

    assert qa(dt=_native.F16) == DTYPE
    assert qa(K=100) == SHAPE
    assert qa(z=0) == INVALID
    assert qa(x=U) == ALIGN
    assert qa(z=A + 2) == ALIGN

    def zt(wp=A, K=256, group=128, zc=A, qmin=-7, colsum=16):
        return lib.w4_zero_point_term(ctypes.c_void_p(wp), ctypes.c_void_p(A), K, 128, group, qmin, colsum,
                                      ctypes.c_void_p(zc), None)

    assert zt(K=200) == SHAPE
    assert zt(group=48) == SHAPE
    assert zt(zc=0) == INVALID
    assert zt(wp=U) == ALIGN
    assert zt(zc=A + 2) == ALIGN
    assert zt(qmin=-6) == INVALID
    assert zt(colsum=-1) == INVALID
    # the asymmetric accumulator's worst case, 255 * |qmin| * group * colsum, must stay below 2^31
    OVERFLOW = 5
    assert zt(colsum=(1 << 31) // (255 * 7 * 128) + 1) == OVERFLOW
    assert zt(colsum=(1 << 31) // (255 * 8 * 128) + 1, qmin=-8) == OVERFLOW
    assert zt(colsum=(1 << 31) // (255 * 8 * 128) + 1, qmin=-8, zc=0) == OVERFLOW  # refused before anything else

    def ga(z=A, zc=A, M=16, dt=_native.F16, alpha=1024):
        return lib.w4a8_gemm_intscale_asym(ctypes.c_void_p(A), ctypes.c_void_p(A), ctypes.c_void_p(z),
                                           ctypes.c_void_p(A), ctypes.c_void_p(A), ctypes.c_void_p(zc), alpha, M, 128,
                                           256, 128, ctypes.c_void_p(A), dt, None, 0, None)

    assert ga(z=0) == INVALID
    assert ga(zc=0) == INVALID
    assert ga(z=A + 2) == ALIGN  # zero points are int32: 4-byte aligned
    assert ga(dt=_native.BF16) == DTYPE
    assert ga(alpha=48) == INVALID
    assert ga(M=0) == OK


def test_failed_gemm_rezeroes_cached_workspaces(lib):
    # host logic: a GEMM that failed or timed out may leave split-tile counts in
    # the cached workspace, so the binding zeroes every cached workspace
    class FakeWs:
        zeroed = 0

        def zero_(self):
            FakeWs.zeroed += 1

    saved = dict(_native._ws_cache)
    try:
        _native._ws_cache.clear()
        _native._ws_cache[0] = FakeWs()
        with pytest.raises(_native.W4A8Error):
            _native._check("w4a8_gemm_intscale", 8)  # W4A8_ERR_TIMEOUT
        assert FakeWs.zeroed == 1
        with pytest.raises(_native.W4A8Error):
            _native._check("w4a8_gemm_intscale", 2)  # a shape error launches nothing
        assert FakeWs.zeroed == 1
    finally:
        _native._ws_cache.clear()
        _native._ws_cache.update(saved)


def test_grouped_argument_checks(lib):
    def gr(E=4, R=16, T=8, dt=_native.F16, alpha=1024, K=256, q=A, off=A, wp=A, sp=A, out_row=0, y_rows=16, y=A):
        return lib.w4a8_gemm_intscale_grouped(ctypes.c_void_p(q), ctypes.c_void_p(A), T, ctypes.c_void_p(A),
                                              ctypes.c_void_p(off), ctypes.c_void_p(out_row), ctypes.c_void_p(wp),
                                              ctypes.c_void_p(sp), alpha, E, R, 128, K, 128, ctypes.c_void_p(y), dt,
                                              y_rows, None, 0, None)

    assert gr(E=0) == INVALID
    assert gr(E=257) == INVALID
    assert gr(K=200) == SHAPE
    assert gr(R=-1) == SHAPE
    assert gr(dt=_native.BF16) == DTYPE
    assert gr(alpha=6) == INVALID
    assert gr(R=0) == OK  # nothing routed: a no-op
    assert gr(T=0) == SHAPE
    assert gr(y_rows=15) == SHAPE  # rows written in routed order need y_rows >= R
    assert gr(q=0) == INVALID
    assert gr(wp=0) == INVALID
    assert gr(q=U) == ALIGN
    assert gr(off=A + 4) == ALIGN  # int64 offsets: 8-byte aligned
    assert gr(sp=A + 4) == ALIGN
    assert lib.w4a8_grouped_workspace_size(0, 128, 256, 128) == -1
    assert lib.w4a8_grouped_workspace_size(4, 100, 256, 128) == -1
