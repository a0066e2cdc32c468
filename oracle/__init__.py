"""CPU oracle for the W4A8 Integer-Scale linear layer (TEST INFRASTRUCTURE).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never calls it and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain scalar C, int64 accumulation, fp64
results); this module compiles it with gcc on first use (or ``build()``) and
wraps each function with numpy marshalling.  Every function cites the passage
it follows in the C source.  Two small steps are written here in numpy because
they are plain definitions: the unquantized fp64 matmul ``x @ w`` used as the
accuracy reference, and rounding an fp64 result to the output type.

Parity status per function (what pins it, see tests/test_oracle_pins.py):
  quantize_rows_asym               hand-worked golden row, brute-force nearest code on
                                   the grid s (q - z), zero exactly representable,
                                   |x - s (q - z)| <= s/2 on rows spanning zero, the
                                   range ends at the extreme codes, constant rows
  intscale_acc_asym                equals intscale_acc when z = 0; equals the expanded
                                   form q_W q_X - Z_X q_W (numpy int64); brute fp64
                                   dequantized matmul on tiny inputs
  quantize_groups(qmin=-8)         brute-force nearest code in [-8, 7], the negative
                                   extreme at -8, positive clipping, error bounds
  quantize_rows / quantize_groups  brute-force nearest-code search, tie cases,
                                   round-trip error bound |x - s q| <= s/2,
                                   error variance ~ s^2/12, hand-worked goldens
  pack_int4 / unpack_int4          exhaustive nibble round trip, hand-packed bytes
  amplifier_search                 postcondition (min scale * alpha >= 1 and
                                   minimal), frexp closed form, hand-worked goldens
  integer_scales                   |S - s*alpha| <= 1/2, exact at representable values
  alpha_sweep                      MSE <= mean(q^2) / (4 alpha^2), zero when every
                                   s_g * alpha is an integer, a hand-worked case,
                                   bit counts at powers of two
  intscale_acc                     equals the expanded-W_int form, numpy int64
                                   matmul when S is constant over groups, brute
                                   fp64 dequantized matmul on tiny inputs, X=0,
                                   one-hot columns
  floatscale                       equals the per-channel outer-product dequant
                                   when group = K; equals intscale when s_g*alpha
                                   is an integer
  moe_intscale                     one expert with every token routed to it is the
                                   dense layer; identical experts repeat the dense
                                   rows; the shared amplifier's postcondition over
                                   all experts; rows depend only on (token, expert)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

INT8_QMAX = 127
INT4_QMAX = 7
INT8_ASYM_QMIN = -128
INT8_ASYM_QMAX = 127


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with plain IEEE floating point."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = [
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
            "-ffp-contract=off", "-o", _LIB, _SRC, "-lm",
        ]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I = ctypes.c_int64
            I32 = ctypes.c_int32
            sig = {
                "oracle_quantize_rows": ([P, I, I, I32, P, P], None),
                "oracle_quantize_rows_asym": ([P, I, I, I32, I32, P, P, P], None),
                "oracle_quantize_groups": ([P, I, I, I, I32, P, P], None),
                "oracle_quantize_groups_full_range": ([P, I, I, I, P, P], None),
                "oracle_pack_int4": ([P, I, I, P], None),
                "oracle_alpha_sweep": ([P, P, I, I, I, P, I, P, P], None),
                "oracle_unpack_int4": ([P, I, I, P], None),
                "oracle_amplifier_search": ([P, I], I32),
                "oracle_integer_scales": ([P, I, I32, P], None),
                "oracle_intscale_acc": ([P, P, P, I, I, I, I, P], I),
                "oracle_intscale_acc_expanded": ([P, P, P, I, I, I, I, P], None),
                "oracle_intscale_acc_at": ([P, P, P, I, I, I, I, P, P, I, P], I),
                "oracle_intscale_acc_asym": ([P, P, P, P, I, I, I, I, P], I),
                "oracle_intscale_output": ([P, P, I32, I, I, P], None),
                "oracle_floatscale": ([P, P, P, P, I, I, I, I, P], None),
                "oracle_floatscale_at": ([P, P, P, P, I, I, I, I, P, P, I, P], None),
                "oracle_scale_colsum_max": ([P, I, I], I),
            }
            for name, (args, res) in sig.items():
                f = getattr(lib, name)
                f.argtypes = args
                f.restype = res
            _lib = lib
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- quantizers

def quantize_rows(x, qmax: int = INT8_QMAX):
    """Per-row symmetric quantization: returns (q int8 [R,C], s float32 [R])."""
    x = _c(x, np.float32)
    R, C = x.shape
    q = np.empty((R, C), np.int8)
    s = np.empty(R, np.float32)
    _load().oracle_quantize_rows(_p(x), R, C, qmax, _p(q), _p(s))
    return q, s


def quantize_act_per_token(x):
    """Per-token int8 activation codes and scales (qmax = 127)."""
    return quantize_rows(x, INT8_QMAX)


def quantize_rows_asym(x, qmin: int = INT8_ASYM_QMIN, qmax: int = INT8_ASYM_QMAX):
    """Per-row asymmetric quantization: returns (q int8 [R,C], s float32 [R], z int32 [R])."""
    x = _c(x, np.float32)
    R, C = x.shape
    q = np.empty((R, C), np.int8)
    s = np.empty(R, np.float32)
    z = np.empty(R, np.int32)
    _load().oracle_quantize_rows_asym(_p(x), R, C, int(qmin), int(qmax), _p(q), _p(s), _p(z))
    return q, s, z


def quantize_act_per_token_asym(x):
    """Per-token asymmetric int8 activation codes in [-128, 127], scales and zero points."""
    return quantize_rows_asym(x, INT8_ASYM_QMIN, INT8_ASYM_QMAX)


def quantize_groups(w, group: int = 128, qmax: int = INT4_QMAX, qmin: int | None = None):
    """Per-(group, column) symmetric quantization of w [K,N]: (q int8 [K,N], s_g float32 [K/group,N]).
    qmin=None: codes in [-qmax, qmax], s = max|w| / qmax.  qmin=-8 (with qmax 7):
    the full int4 range [-8, 7], s = max|w| / 8."""
    w = _c(w, np.float32)
    K, N = w.shape
    if K % group:
        raise ValueError("K must be a multiple of group")
    q = np.empty((K, N), np.int8)
    s = np.empty((K // group, N), np.float32)
    if qmin is None or qmin == -qmax:
        _load().oracle_quantize_groups(_p(w), K, N, group, qmax, _p(q), _p(s))
    elif qmin == -8 and qmax == 7:
        _load().oracle_quantize_groups_full_range(_p(w), K, N, group, _p(q), _p(s))
    else:
        raise ValueError(f"unsupported code range [{qmin}, {qmax}]")
    return q, s


def pack_int4(q):
    """Codes q [K,N] in [-8,7] -> packed uint8 [N, K/2] (K a multiple of 8)."""
    q = _c(q, np.int8)
    K, N = q.shape
    if K % 8:
        raise ValueError(f"K must be a multiple of 8, got {K}")
    out = np.empty((N, K // 2), np.uint8)
    _load().oracle_pack_int4(_p(q), K, N, _p(out))
    return out


def unpack_int4(packed, K: int, N: int):
    if K % 8:
        raise ValueError(f"K must be a multiple of 8, got {K}")
    packed = _c(packed, np.uint8)
    out = np.empty((K, N), np.int8)
    _load().oracle_unpack_int4(_p(packed), K, N, _p(out))
    return out


def amplifier_search(scales) -> int:
    s = _c(np.ravel(scales), np.float32)
    return int(_load().oracle_amplifier_search(_p(s), s.size))


def integer_scales(s_g, alpha: int):
    s = _c(s_g, np.float32)
    out = np.empty(s.shape, np.int32)
    _load().oracle_integer_scales(_p(s), s.size, int(alpha), _p(out))
    return out


def alpha_sweep(qw, s_g, alphas, group: int = 128):
    """Amplifier analysis (Integer Scale summary §4, Fig. 4(a)/(c)): for each
    alpha, the weight MSE between integer-scale (S / alpha) and float-scale
    (s_g) dequantization of the codes qw [K,N], and the bits of the largest
    S = rne(s_g * alpha).  Returns (mse [n] float64, bits [n] int32)."""
    qw = _c(qw, np.int8)
    s_g = _c(s_g, np.float32)
    a = _c(np.ravel(alphas), np.int32)
    K, N = qw.shape
    mse = np.empty(a.size, np.float64)
    bits = np.empty(a.size, np.int32)
    _load().oracle_alpha_sweep(_p(qw), _p(s_g), K, N, group, _p(a), a.size, _p(mse), _p(bits))
    return mse, bits


def scale_colsum_max(S) -> int:
    S = _c(S, np.int32)
    G, N = S.shape
    return int(_load().oracle_scale_colsum_max(_p(S), G, N))


# ---------------------------------------------------------------- GEMMs

class Int32BoundError(ValueError):
    """An integer accumulator of the layer does not fit the int32 range the
    kernels accumulate in (the Integer Scale summary, §4: the amplifier stays
    at 1024 so that integer accumulation does not overflow)."""


def _int32_checked(bad: int, what: str):
    if bad:
        raise Int32BoundError(f"{what}: {bad} accumulator(s) outside the int32 range")


def check_worst_case(S, group: int, qx_max: int = INT8_QMAX, qw_max: int = INT4_QMAX):
    """Raise Int32BoundError unless qx_max * qw_max * group * max_n sum_g |S[g,n]|
    < 2^31: then no input whatever can push an accumulator out of int32."""
    worst = int(qx_max) * int(qw_max) * int(group) * scale_colsum_max(S)
    if worst >= 1 << 31:
        raise Int32BoundError(f"worst-case accumulator {worst} >= 2^31")


def intscale_acc(qx, qw, S, group: int = 128):
    """Raw integer-scale accumulators acc [M, N] (int64); raises
    Int32BoundError when any of them lies outside (-2^31, 2^31)."""
    qx = _c(qx, np.int8)
    qw = _c(qw, np.int8)
    S = _c(S, np.int32)
    M, K = qx.shape
    N = qw.shape[1]
    acc = np.empty((M, N), np.int64)
    _int32_checked(_load().oracle_intscale_acc(_p(qx), _p(qw), _p(S), M, N, K, group, _p(acc)), "intscale_acc")
    return acc


def intscale_acc_expanded(qx, qw, S, group: int = 128):
    qx = _c(qx, np.int8)
    qw = _c(qw, np.int8)
    S = _c(S, np.int32)
    M, K = qx.shape
    N = qw.shape[1]
    acc = np.empty((M, N), np.int64)
    _load().oracle_intscale_acc_expanded(_p(qx), _p(qw), _p(S), M, N, K, group, _p(acc))
    return acc


def intscale_acc_at(qx, qw, S, ms, ns, group: int = 128):
    qx = _c(qx, np.int8)
    qw = _c(qw, np.int8)
    S = _c(S, np.int32)
    ms = _c(ms, np.int64)
    ns = _c(ns, np.int64)
    M, K = qx.shape
    N = qw.shape[1]
    acc = np.empty(ms.size, np.int64)
    _int32_checked(_load().oracle_intscale_acc_at(_p(qx), _p(qw), _p(S), M, N, K, group, _p(ms), _p(ns), ms.size,
                                                  _p(acc)), "intscale_acc_at")
    return acc


def intscale_acc_asym(qx, z, qw, S, group: int = 128):
    qx = _c(qx, np.int8)
    z = _c(z, np.int32)
    qw = _c(qw, np.int8)
    S = _c(S, np.int32)
    M, K = qx.shape
    N = qw.shape[1]
    acc = np.empty((M, N), np.int64)
    _int32_checked(_load().oracle_intscale_acc_asym(_p(qx), _p(z), _p(qw), _p(S), M, N, K, group, _p(acc)),
                   "intscale_acc_asym")
    return acc


def intscale_output(acc, s_a, alpha: int):
    acc = _c(acc, np.int64)
    s_a = _c(s_a, np.float32)
    M, N = acc.shape
    y = np.empty((M, N), np.float64)
    _load().oracle_intscale_output(_p(acc), _p(s_a), int(alpha), M, N, _p(y))
    return y


def floatscale(qx, s_a, qw, s_g, group: int = 128):
    qx = _c(qx, np.int8)
    s_a = _c(s_a, np.float32)
    qw = _c(qw, np.int8)
    s_g = _c(s_g, np.float32)
    M, K = qx.shape
    N = qw.shape[1]
    y = np.empty((M, N), np.float64)
    _load().oracle_floatscale(_p(qx), _p(s_a), _p(qw), _p(s_g), M, N, K, group, _p(y))
    return y


def floatscale_at(qx, s_a, qw, s_g, ms, ns, group: int = 128):
    qx = _c(qx, np.int8)
    s_a = _c(s_a, np.float32)
    qw = _c(qw, np.int8)
    s_g = _c(s_g, np.float32)
    ms = _c(ms, np.int64)
    ns = _c(ns, np.int64)
    M, K = qx.shape
    N = qw.shape[1]
    y = np.empty(ms.size, np.float64)
    _load().oracle_floatscale_at(_p(qx), _p(s_a), _p(qw), _p(s_g), M, N, K, group, _p(ms), _p(ns), ms.size, _p(y))
    return y


def round_output(y, out: str):
    """fp64 result -> the output type ('f32' or 'f16'), round to nearest even."""
    if out == "f32":
        return np.asarray(y, np.float64).astype(np.float32)
    if out == "f16":
        return np.asarray(y, np.float64).astype(np.float16)
    raise ValueError(out)


# ---------------------------------------------------------------- whole layer

def linear_intscale(x, w, *, group: int = 128, alpha=1024, out: str = "f16", qmin: int | None = None,
                    wbits: int = 4, asym: bool = False):
    """The whole Integer-Scale path on the CPU.

    alpha: an integer power of two, or None for the amplifier search.
    qmin: None for weight codes in [-7, 7], -8 for the full int4 range.
    wbits: 4 (int4 codes, nibble-packed) or 8 (W8A8: codes in [-127, 127],
    s_g = max|w| / 127, 'packed' is then the int8 layout w8 [N, K]).
    asym: asymmetric per-token activations (codes in [-128, 127] with a zero
    point z per token; the accumulator is then sum_g S sum_k (qx - z) qw).
    Returns a dict with every intermediate (codes, scales, zero points, packed
    bytes, integer scales, raw accumulators, fp64 and rounded outputs).
    """
    if asym:
        qx, s_a, z = quantize_act_per_token_asym(x)
    else:
        qx, s_a = quantize_act_per_token(x)
        z = np.zeros(qx.shape[0], np.int32)
    if wbits == 8:
        qw, s_g = quantize_groups(w, group, qmax=INT8_QMAX)
    else:
        qw, s_g = quantize_groups(w, group, qmin=qmin)
    a = amplifier_search(s_g) if alpha is None else int(alpha)
    S = integer_scales(s_g, a)
    # the worst case over every input the layer may see must fit in int32
    # (the column bound the pack step checks): widest |code| of each operand
    # times group times the largest column sum of |S|
    qx_max = 255 if asym else INT8_QMAX
    qw_max = INT8_QMAX if wbits == 8 else (8 if qmin == -8 else INT4_QMAX)
    check_worst_case(S, group, qx_max, qw_max)
    acc = intscale_acc_asym(qx, z, qw, S, group) if asym else intscale_acc(qx, qw, S, group)
    y64 = intscale_output(acc, s_a, a)
    packed = np.ascontiguousarray(qw.T) if wbits == 8 else pack_int4(qw)
    return dict(qx=qx, s_a=s_a, z=z, qw=qw, s_g=s_g, packed=packed, alpha=a, S=S, acc=acc,
                y64=y64, y=round_output(y64, out))


def linear_floatscale(x, w, *, group: int = 128, out: str = "f16"):
    qx, s_a = quantize_act_per_token(x)
    qw, s_g = quantize_groups(w, group)
    y64 = floatscale(qx, s_a, qw, s_g, group)
    return dict(qx=qx, s_a=s_a, qw=qw, s_g=s_g, y64=y64, y=round_output(y64, out))


# ---------------------------------------------------------------- mixture of experts

def moe_intscale(x, ws, row_index, offsets, *, group: int = 128, alpha=1024, out: str = "f16"):
    """A mixture-of-experts layer through the Integer-Scale path (the Integer
    Scale summary, the Mixtral results of §5.3: per-expert fine-grained W4A8
    GEMMs).  Every token is quantized once (its scale does not depend on the
    expert); the amplifier is one per layer (the search of §3.3 run over the
    group scales of all experts: the layer spans all of them, a reading); the
    routed rows of expert e, row_index[offsets[e]:offsets[e+1]], go through
    expert e's integer-scale GEMM.

    Returns the routed rows' raw accumulators acc [R, N], fp64 outputs y64,
    the rounded outputs, the shared alpha and every expert's codes, scales,
    packed bytes and integer scales.
    """
    qx, s_a = quantize_act_per_token(x)
    qws, sgs = [], []
    for w in ws:
        qw, sg = quantize_groups(w, group)
        qws.append(qw)
        sgs.append(sg)
    a = amplifier_search(np.concatenate([sg.reshape(-1) for sg in sgs])) if alpha is None else int(alpha)
    Ss = [integer_scales(sg, a) for sg in sgs]
    for S in Ss:
        check_worst_case(S, group)
    row_index = np.asarray(row_index, np.int64)
    N = ws[0].shape[1]
    acc = np.zeros((row_index.shape[0], N), np.int64)
    y64 = np.zeros((row_index.shape[0], N), np.float64)
    for e in range(len(ws)):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        toks = row_index[lo:hi]
        acc[lo:hi] = intscale_acc(qx[toks], qws[e], Ss[e], group)
        y64[lo:hi] = intscale_output(acc[lo:hi], s_a[toks], a)
    return dict(qx=qx, s_a=s_a, qw=qws, s_g=sgs, S=Ss, packed=[pack_int4(q) for q in qws], alpha=a, acc=acc,
                y64=y64, y=round_output(y64, out))

