"""ctypes binding of the C ABI in include/w4a8_intscale.h.

Argument marshalling only: torch tensors are checked for device, dtype,
shape and contiguity, and their data pointers and the current CUDA stream are
handed to the library, which does every step of the computation in its own
kernels.  There is no CPU path: a missing library or a CPU tensor raises.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libw4a8_intscale.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "w4a8_intscale.h")

# w4a8_dtype
F32, F16, BF16, I32 = 0, 1, 2, 3
PACK_WORKSPACE_BYTES = 1 << 20

STATUS = {
    0: "W4A8_OK",
    1: "W4A8_ERR_INVALID_ARG",
    2: "W4A8_ERR_SHAPE",
    3: "W4A8_ERR_ALIGN",
    4: "W4A8_ERR_DTYPE",
    5: "W4A8_ERR_OVERFLOW_BOUND",
    6: "W4A8_ERR_SCALE_RANGE",
    7: "W4A8_ERR_CUDA",
    8: "W4A8_ERR_TIMEOUT",
    9: "W4A8_ERR_WORKSPACE",
}


class W4A8Error(RuntimeError):
    def __init__(self, fn: str, code: int, detail: str = ""):
        self.code = code
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}{detail}")


_lock = threading.Lock()
_lib = None


def declared_symbols():
    """Names of the functions the public header declares."""
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"W4A8_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def load(path: str = LIB_PATH):
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(
                f"CUDA library not found at {path}; build it with `python -m bit_gemm_quantize_b200.build`"
            )
        lib = ctypes.CDLL(path)
        P, I64, I32_ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
        sigs = {
            "w4a8_status_string": ([I32_], ctypes.c_char_p),
            "quantize_act_per_token": ([P, I32_, I64, I64, I64, P, P, P], I32_),
            "quantize_act_routed": ([P, I32_, I64, I64, I64, P, I64, P, P, P], I32_),
            "quantize_act_per_token_asym": ([P, I32_, I64, I64, I64, P, P, P, P], I32_),
            "w4_zero_point_term": ([P, P, I64, I64, I32_, I32_, I64, P, P], I32_),
            "w4a8_static_workspace_reset": ([], I32_),
            "w4a8_gemm_intscale_asym": ([P, P, P, P, P, P, I32_, I64, I64, I64, I32_, P, I32_, P, I64, P], I32_),
            "w4a8_amplifier_search": ([P, I64, P, P, P], I32_),
            "pack_w4_groupwise": ([P, I64, I64, I32_, I32_, P, P, P, P, P, P, P], I32_),
            "pack_w4_groupwise_range": ([P, I64, I64, I32_, I32_, I32_, P, P, P, P, P, P, P], I32_),
            "pack_w8_groupwise": ([P, I64, I64, I32_, I32_, P, P, P, P, P, P, P], I32_),
            "w8a8_gemm_intscale": ([P, P, P, P, I32_, I64, I64, I64, I32_, P, I32_, P, I64, P], I32_),
            "w4a8_gemm_workspace_size": ([I64, I64, I64, I32_, I32_], I64),
            "w4a8_gemm_intscale": ([P, P, P, P, I32_, I64, I64, I64, I32_, P, I32_, P, I64, P], I32_),
            "w4a8_gemm_intscale_static_ws": ([P, P, P, P, I32_, I64, I64, I64, I32_, P, I32_, P], I32_),
            "w4a8_gemm_floatscale": ([P, P, P, P, I64, I64, I64, I32_, P, I32_, P, I64, P], I32_),
            "w4a8_device_status": ([P, I32_], I32_),
            "w4a8_linear_intscale": ([P, I32_, I64, I64, I64, P, P, I32_, I64, I32_, P, I32_, P, P, P, I64, P], I32_),
            "w4a8_grouped_workspace_size": ([I32_, I64, I64, I32_], I64),
            "w4a8_gemm_intscale_grouped": ([P, P, I64, P, P, P, P, P, I32_, I32_, I64, I64, I64, I32_, P, I32_, I64,
                                            P, I64, P], I32_),
            "w4a8_tensor_i8_peak_probe": ([I64, I32_, I32_, P, P, P], I32_),
            "w4a8_set_wait_limit": ([I64], I64),
            "w4a8_last_cuda_error": ([I32_], I32_),
            "w4a8_cuda_error_string": ([I32_], ctypes.c_char_p),
        }
        for name, (args, res) in sigs.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
        return lib


def _check(fn: str, code: int):
    if code != 0:
        if "gemm" in fn and code in (7, 8):  # a launch failed: its workspace may hold counts
            _reset_workspaces()
        detail = ""
        if code == 7:  # W4A8_ERR_CUDA: name the runtime error behind it
            lib = load()
            e = int(lib.w4a8_last_cuda_error(1))
            detail = f" ({lib.w4a8_cuda_error_string(e).decode()})"
        raise W4A8Error(fn, code, detail)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need_cuda(name, t, dtype=None, ndim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


# ------------------------------------------------------------------ workspace

_ws_cache = {}


_static_ws_devices = set()  # devices on which the library's own workspace has been used


def _reset_workspaces():
    """Zero every cached GEMM workspace and the library's own (static)
    workspace counters: after a failed launch or a device-side error the
    split-tile arrival counters may be left nonzero."""
    for ws in _ws_cache.values():
        try:
            ws.zero_()
        except Exception:  # a lost context: nothing more to clean
            pass
    for d in list(_static_ws_devices):
        try:
            with torch.cuda.device(d):
                load().w4a8_static_workspace_reset()
        except Exception:
            pass


def gemm_workspace(M: int, N: int, K: int, group: int, path: int, device) -> torch.Tensor | None:
    """A zero-filled workspace big enough for the call, reused across calls on
    the device (the kernels leave it zeroed after a successful call).  Calls
    that may overlap on the GPU (different streams without ordering) must
    each pass a workspace of their own."""
    lib = load()
    with torch.cuda.device(device):
        need = int(lib.w4a8_gemm_workspace_size(M, N, K, group, path))
    if need < 0:
        raise RuntimeError("w4a8_gemm_workspace_size: no CUDA device")
    if need == 0:
        return None
    key = torch.device(device).index
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(need, dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


# ------------------------------------------------------------------ operations

def quantize_act_per_token(x: torch.Tensor, q_x: torch.Tensor | None = None, s_a: torch.Tensor | None = None):
    """Per-token int8 codes and fp32 scales of x [M, K] (fp32 or bf16)."""
    _need_cuda("x", x, ndim=2)
    if x.dtype == torch.float32:
        dt = F32
    elif x.dtype == torch.bfloat16:
        dt = BF16
    else:
        raise ValueError("x must be float32 or bfloat16")
    M, K = x.shape
    if q_x is None:
        q_x = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if s_a is None:
        s_a = torch.empty((M,), dtype=torch.float32, device=x.device)
    _need_cuda("q_x", q_x, torch.int8, 2)
    _need_cuda("s_a", s_a, torch.float32, 1)
    code = load().quantize_act_per_token(_ptr(x), dt, M, K, K, _ptr(q_x), _ptr(s_a), _stream(x.device))
    _check("quantize_act_per_token", code)
    return q_x, s_a


def quantize_act_routed(x: torch.Tensor, row_index: torch.Tensor, q_r: torch.Tensor | None = None,
                        s_r: torch.Tensor | None = None):
    """Per-token int8 codes and scales of x [T, K] in routed order: row i is
    token row_index[i] ([R] int32 on the device)."""
    _need_cuda("x", x, ndim=2)
    if x.dtype == torch.float32:
        dt = F32
    elif x.dtype == torch.bfloat16:
        dt = BF16
    else:
        raise ValueError("x must be float32 or bfloat16")
    _need_cuda("row_index", row_index, torch.int32, 1)
    T, K = x.shape
    R = row_index.shape[0]
    if q_r is None:
        q_r = torch.empty((R, K), dtype=torch.int8, device=x.device)
    if s_r is None:
        s_r = torch.empty((R,), dtype=torch.float32, device=x.device)
    _need_cuda("q_r", q_r, torch.int8, 2)
    _need_cuda("s_r", s_r, torch.float32, 1)
    code = load().quantize_act_routed(_ptr(x), dt, T, K, K, _ptr(row_index), R, _ptr(q_r), _ptr(s_r),
                                      _stream(x.device))
    _check("quantize_act_routed", code)
    return q_r, s_r


def w4a8_amplifier_search(scales: torch.Tensor) -> int:
    _need_cuda("scales", scales, torch.float32)
    ws = torch.empty(PACK_WORKSPACE_BYTES, dtype=torch.uint8, device=scales.device)
    alpha = ctypes.c_int32(0)
    code = load().w4a8_amplifier_search(_ptr(scales), scales.numel(), _ptr(ws), ctypes.byref(alpha),
                                        _stream(scales.device))
    _check("w4a8_amplifier_search", code)
    return int(alpha.value)


def pack_w4_groupwise(w: torch.Tensor, group: int = 128, alpha: int | None = 1024, scales_only: bool = False,
                      qmin: int = -7):
    """Quantize and pack fp32 weights w [K, N].  alpha=None runs the search.
    qmin=-7: codes in [-7, 7], s_g = max|w| / 7; qmin=-8: the full int4
    range [-8, 7], s_g = max|w| / 8.

    Returns dict(packed [N, K/2] uint8, s_g [K/group, N] f32, S [K/group, N]
    int16, alpha, colsum_max), or dict(s_g) when scales_only."""
    _need_cuda("w", w, torch.float32, 2)
    K, N = w.shape
    dev = w.device
    s_g = torch.empty((K // group, N), dtype=torch.float32, device=dev)
    ws = torch.empty(PACK_WORKSPACE_BYTES, dtype=torch.uint8, device=dev)
    lib = load()
    if scales_only:
        code = lib.pack_w4_groupwise_range(_ptr(w), K, N, group, 0, int(qmin), None, _ptr(s_g), None, None, None,
                                           _ptr(ws), _stream(dev))
        _check("pack_w4_groupwise_range", code)
        return dict(s_g=s_g)
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    S = torch.empty((K // group, N), dtype=torch.int16, device=dev)
    a_out = ctypes.c_int32(0)
    colsum = ctypes.c_int64(0)
    code = lib.pack_w4_groupwise_range(_ptr(w), K, N, group, 0 if alpha is None else int(alpha), int(qmin),
                                       _ptr(packed), _ptr(s_g), _ptr(S), ctypes.byref(a_out), ctypes.byref(colsum),
                                       _ptr(ws), _stream(dev))
    _check("pack_w4_groupwise_range", code)
    return dict(packed=packed, s_g=s_g, S=S, alpha=int(a_out.value), colsum_max=int(colsum.value))


def pack_w8_groupwise(w: torch.Tensor, group: int = 128, alpha: int | None = None):
    """Quantize fp32 weights w [K, N] to per-group 8-bit codes (W8A8).
    alpha=None runs the search.  Returns dict(w8 [N, K] int8, s_g [K/group, N]
    f32, S [K/group, N] int16, alpha, colsum_max)."""
    _need_cuda("w", w, torch.float32, 2)
    K, N = w.shape
    dev = w.device
    w8 = torch.empty((N, K), dtype=torch.int8, device=dev)
    s_g = torch.empty((K // group, N), dtype=torch.float32, device=dev)
    S = torch.empty((K // group, N), dtype=torch.int16, device=dev)
    ws = torch.empty(PACK_WORKSPACE_BYTES, dtype=torch.uint8, device=dev)
    a_out = ctypes.c_int32(0)
    colsum = ctypes.c_int64(0)
    code = load().pack_w8_groupwise(_ptr(w), K, N, group, 0 if alpha is None else int(alpha), _ptr(w8), _ptr(s_g),
                                    _ptr(S), ctypes.byref(a_out), ctypes.byref(colsum), _ptr(ws), _stream(dev))
    _check("pack_w8_groupwise", code)
    return dict(w8=w8, s_g=s_g, S=S, alpha=int(a_out.value), colsum_max=int(colsum.value))


_OUT = {"f32": (F32, torch.float32), "f16": (F16, torch.float16), "i32": (I32, torch.int32)}


def quantize_act_per_token_asym(x: torch.Tensor, q_x: torch.Tensor | None = None,
                                s_a: torch.Tensor | None = None, z_a: torch.Tensor | None = None):
    """Per-token asymmetric int8 codes in [-128, 127], fp32 scales and int32
    zero points of x [M, K] (fp32 or bf16)."""
    _need_cuda("x", x, ndim=2)
    if x.dtype == torch.float32:
        dt = F32
    elif x.dtype == torch.bfloat16:
        dt = BF16
    else:
        raise ValueError("x must be float32 or bfloat16")
    M, K = x.shape
    if q_x is None:
        q_x = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if s_a is None:
        s_a = torch.empty((M,), dtype=torch.float32, device=x.device)
    if z_a is None:
        z_a = torch.empty((M,), dtype=torch.int32, device=x.device)
    _need_cuda("q_x", q_x, torch.int8, 2)
    _need_cuda("s_a", s_a, torch.float32, 1)
    _need_cuda("z_a", z_a, torch.int32, 1)
    code = load().quantize_act_per_token_asym(_ptr(x), dt, M, K, K, _ptr(q_x), _ptr(s_a), _ptr(z_a),
                                              _stream(x.device))
    _check("quantize_act_per_token_asym", code)
    return q_x, s_a, z_a


def w4_zero_point_term(w_packed: torch.Tensor, S: torch.Tensor, group: int = 128, *, colsum_max: int | None = None,
                       qmin: int = -7) -> torch.Tensor:
    """zc [N] int32 = sum_g S[g, n] * sum_{k in g} q[k, n] from the packed codes
    (the weight-side term of an asymmetric activation's zero point).
    colsum_max: max_n sum_g |S[g, n]| as the pack reported it (taken from S
    when not given); the library refuses weights whose asymmetric accumulator
    could leave int32 (W4A8_ERR_OVERFLOW_BOUND)."""
    _need_cuda("w_packed", w_packed, torch.uint8, 2)
    _need_cuda("S", S, torch.int16, 2)
    N, K2 = w_packed.shape
    K = 2 * K2
    if S.shape != (K // group, N):
        raise ValueError("S must be [K / group, N]")
    if colsum_max is None:
        colsum_max = int(S.abs().to(torch.int64).sum(0).max().item())
    zc = torch.empty((N,), dtype=torch.int32, device=w_packed.device)
    code = load().w4_zero_point_term(_ptr(w_packed), _ptr(S), K, N, group, int(qmin), int(colsum_max), _ptr(zc),
                                     _stream(w_packed.device))
    _check("w4_zero_point_term", code)
    return zc


def _gemm_args(q_x, s_a, packed, N, K, group):
    _need_cuda("q_x", q_x, torch.int8, 2)
    _need_cuda("s_a", s_a, torch.float32, 1)
    _need_cuda("w_packed", packed, torch.uint8, 2)
    M = q_x.shape[0]
    if q_x.shape[1] != K or packed.shape != (N, K // 2) or s_a.shape[0] != M:
        raise ValueError("inconsistent GEMM operand shapes")
    return M


def w4a8_gemm_intscale(q_x, s_a, w_packed, S, alpha: int, *, group: int = 128, out: str = "f16",
                       y: torch.Tensor | None = None, workspace: torch.Tensor | None = None):
    """y [M, N] = integer-scale W4A8 GEMM (out: 'f16', 'f32' or 'i32' raw accumulators)."""
    N, K2 = w_packed.shape
    K = 2 * K2
    M = _gemm_args(q_x, s_a, w_packed, N, K, group)
    _need_cuda("S", S, torch.int16, 2)
    dt, tdt = _OUT[out]
    if y is None:
        y = torch.empty((M, N), dtype=tdt, device=q_x.device)
    _need_cuda("y", y, tdt, 2)
    if workspace is None:
        workspace = gemm_workspace(M, N, K, group, 0, q_x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    code = load().w4a8_gemm_intscale(_ptr(q_x), _ptr(s_a), _ptr(w_packed), _ptr(S), int(alpha), M, N, K, group,
                                     _ptr(y), dt, _ptr(workspace), ws_bytes, _stream(q_x.device))
    _check("w4a8_gemm_intscale", code)
    return y


def w4a8_linear_intscale(x, w_packed, S, alpha: int, *, group: int = 128, out: str = "f16",
                         y: torch.Tensor | None = None, q_x: torch.Tensor | None = None, s_a: torch.Tensor | None = None,
                         workspace: torch.Tensor | None = None):
    """y [M, N] = the integer-scale layer from unquantized tokens x [M, K]
    (fp32 or bf16): per-token quantization and the W4A8 integer-scale GEMM,
    one kernel for M = 1 (256 <= K <= 16384).  q_x / s_a receive the token
    codes and scales when given (allocated here where the quantizer and the
    GEMM run as two kernels)."""
    _need_cuda("x", x, ndim=2)
    if x.dtype == torch.float32:
        dt_x = F32
    elif x.dtype == torch.bfloat16:
        dt_x = BF16
    else:
        raise ValueError("x must be float32 or bfloat16")
    _need_cuda("w_packed", w_packed, torch.uint8, 2)
    _need_cuda("S", S, torch.int16, 2)
    M, K = x.shape
    N = w_packed.shape[0]
    if w_packed.shape[1] * 2 != K:
        raise ValueError("w_packed must be [N, K/2]")
    dt, tdt = _OUT[out]
    if y is None:
        y = torch.empty((M, N), dtype=tdt, device=x.device)
    _need_cuda("y", y, tdt, 2)
    # buffers for the two-kernel route: more than one token (faster as two
    # kernels from two up), or K outside the decode kernel's range
    two_kernels = M > 1 or K < 256 or K > 16384
    if two_kernels and q_x is None:
        q_x = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if two_kernels and s_a is None:
        s_a = torch.empty((M,), dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = gemm_workspace(M, N, K, group, 0, x.device)
    ws_bytes = 0 if workspace is None else workspace.numel()
    code = load().w4a8_linear_intscale(_ptr(x), dt_x, M, K, K, _ptr(w_packed), _ptr(S), int(alpha), N, group,
                                       _ptr(y), dt, _ptr(q_x), _ptr(s_a), _ptr(workspace), ws_bytes,
                                       _stream(x.device))
    _check("w4a8_linear_intscale", code)
    return y


def w4a8_gemm_intscale_asym(q_x, s_a, z_a, w_packed, S, zc, alpha: int, *, group: int = 128, out: str = "f16",
                            y: torch.Tensor | None = None, workspace: torch.Tensor | None = None):
    """y [M, N] = integer-scale W4A8 GEMM of asymmetric token codes: the
    accumulator is sum_g S sum_k (q_x - z_a) q, computed as the symmetric one
    minus z_a[m] * zc[n] (out: 'f16', 'f32' or 'i32' for that accumulator)."""
    N, K2 = w_packed.shape
    K = 2 * K2
    M = _gemm_args(q_x, s_a, w_packed, N, K, group)
    _need_cuda("S", S, torch.int16, 2)
    _need_cuda("z_a", z_a, torch.int32, 1)
    _need_cuda("zc", zc, torch.int32, 1)
    if z_a.shape[0] != M or zc.shape[0] != N:
        raise ValueError("z_a must be [M] and zc [N]")
    dt, tdt = _OUT[out]
    if y is None:
        y = torch.empty((M, N), dtype=tdt, device=q_x.device)
    _need_cuda("y", y, tdt, 2)
    if workspace is None:
        workspace = gemm_workspace(M, N, K, group, 0, q_x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    code = load().w4a8_gemm_intscale_asym(_ptr(q_x), _ptr(s_a), _ptr(z_a), _ptr(w_packed), _ptr(S), _ptr(zc),
                                          int(alpha), M, N, K, group, _ptr(y), dt, _ptr(workspace), ws_bytes,
                                          _stream(q_x.device))
    _check("w4a8_gemm_intscale_asym", code)
    return y


def w8a8_gemm_intscale(q_x, s_a, w8, S, alpha: int, *, group: int = 128, out: str = "f16",
                       y: torch.Tensor | None = None, workspace: torch.Tensor | None = None):
    """y [M, N] = integer-scale W8A8 GEMM with 8-bit weight codes w8 [N, K]
    (out: 'f16', 'f32' or 'i32' raw accumulators)."""
    _need_cuda("q_x", q_x, torch.int8, 2)
    _need_cuda("s_a", s_a, torch.float32, 1)
    _need_cuda("w8", w8, torch.int8, 2)
    N, K = w8.shape
    M = q_x.shape[0]
    if q_x.shape[1] != K or s_a.shape[0] != M:
        raise ValueError("inconsistent GEMM operand shapes")
    _need_cuda("S", S, torch.int16, 2)
    dt, tdt = _OUT[out]
    if y is None:
        y = torch.empty((M, N), dtype=tdt, device=q_x.device)
    _need_cuda("y", y, tdt, 2)
    if workspace is None:
        workspace = gemm_workspace(M, N, K, group, 2, q_x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    code = load().w8a8_gemm_intscale(_ptr(q_x), _ptr(s_a), _ptr(w8), _ptr(S), int(alpha), M, N, K, group, _ptr(y),
                                     dt, _ptr(workspace), ws_bytes, _stream(q_x.device))
    _check("w8a8_gemm_intscale", code)
    return y


def w4a8_gemm_intscale_static_ws(q_x, s_a, w_packed, S, alpha: int, *, group: int = 128, out: str = "f16",
                                 y: torch.Tensor | None = None):
    """w4a8_gemm_intscale with the library's fixed per-device workspace (no workspace argument)."""
    N, K2 = w_packed.shape
    K = 2 * K2
    M = _gemm_args(q_x, s_a, w_packed, N, K, group)
    _need_cuda("S", S, torch.int16, 2)
    dt, tdt = _OUT[out]
    if y is None:
        y = torch.empty((M, N), dtype=tdt, device=q_x.device)
    _need_cuda("y", y, tdt, 2)
    _static_ws_devices.add(torch.device(q_x.device).index)
    code = load().w4a8_gemm_intscale_static_ws(_ptr(q_x), _ptr(s_a), _ptr(w_packed), _ptr(S), int(alpha), M, N, K,
                                               group, _ptr(y), dt, _stream(q_x.device))
    _check("w4a8_gemm_intscale_static_ws", code)
    return y


def w4a8_gemm_floatscale(q_x, s_a, w_packed, s_g, *, group: int = 128, out: str = "f16",
                         y: torch.Tensor | None = None, workspace: torch.Tensor | None = None):
    """y [M, N] = float-scale W4A8 GEMM (the comparison path; out 'f16' or 'f32')."""
    N, K2 = w_packed.shape
    K = 2 * K2
    M = _gemm_args(q_x, s_a, w_packed, N, K, group)
    _need_cuda("s_g", s_g, torch.float32, 2)
    if out not in ("f16", "f32"):
        raise ValueError("float-scale output must be f16 or f32")
    dt, tdt = _OUT[out]
    if y is None:
        y = torch.empty((M, N), dtype=tdt, device=q_x.device)
    _need_cuda("y", y, tdt, 2)
    if workspace is None:
        workspace = gemm_workspace(M, N, K, group, 1, q_x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    code = load().w4a8_gemm_floatscale(_ptr(q_x), _ptr(s_a), _ptr(w_packed), _ptr(s_g), M, N, K, group, _ptr(y),
                                       dt, _ptr(workspace), ws_bytes, _stream(q_x.device))
    _check("w4a8_gemm_floatscale", code)
    return y


def pack_moe_experts(ws, group: int = 128, alpha: int | None = None):
    """Pack every expert's fp32 weights [K, N] with one amplifier for the layer:
    the search over all experts' group scales (alpha=None) or the given one.

    Returns dict(packed=[...], S=[...], s_g=[...], alpha)."""
    if alpha is None:
        sgs = [pack_w4_groupwise(w, group=group, scales_only=True)["s_g"] for w in ws]
        alpha = w4a8_amplifier_search(torch.cat([s.reshape(-1) for s in sgs]))
    pks = [pack_w4_groupwise(w, group=group, alpha=alpha) for w in ws]
    return dict(packed=[p["packed"] for p in pks], S=[p["S"] for p in pks], s_g=[p["s_g"] for p in pks],
                alpha=int(alpha))


_grouped_ws = {}


def grouped_workspace(E: int, N: int, K: int, group: int, device) -> torch.Tensor:
    """A zero-filled workspace for w4a8_gemm_intscale_grouped, reused across
    calls on the device (calls that may overlap on the GPU need their own)."""
    with torch.cuda.device(device):
        need = int(load().w4a8_grouped_workspace_size(int(E), int(N), int(K), int(group)))
    if need < 0:
        raise W4A8Error("w4a8_grouped_workspace_size", 1, " (invalid shape or expert count)")
    key = torch.device(device).index
    ws = _grouped_ws.get(key)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(need, dtype=torch.uint8, device=device)
        _grouped_ws[key] = ws
        _ws_cache[("grouped", key)] = ws  # zeroed with the others after a failure
    return ws


def device_pointers(tensors, device) -> torch.Tensor:
    """A device int64 array of the tensors' data pointers (0 for None): the
    pointer arrays the grouped call reads on the device."""
    ptrs = [0 if t is None else int(t.data_ptr()) for t in tensors]
    return torch.tensor(ptrs, dtype=torch.int64).to(device)


def w4a8_gemm_intscale_grouped(q_x, s_a, row_index, expert_offsets, packed, S, alpha: int, *, group: int = 128,
                               out: str = "f16", y: torch.Tensor | None = None, out_row: torch.Tensor | None = None,
                               y_rows: int | None = None, workspace: torch.Tensor | None = None,
                               N: int | None = None):
    """Every expert's integer-scale GEMM over its routed rows in one grouped call.

    row_index [R] int32: the token of each routed row, rows grouped by expert,
    or None when q_x / s_a are the routed rows themselves (quantize_act_routed);
    expert_offsets [E+1] int64 CUDA tensor (device offsets); packed / S: lists
    of per-expert tensors (None for experts without rows) or int64 CUDA
    tensors of device pointers; out_row [R] int32 or None: the output row of
    each routed row (None: row i).  N is taken from the packed weights unless
    given (needed when pointers are passed)."""
    _need_cuda("q_x", q_x, torch.int8, 2)
    _need_cuda("s_a", s_a, torch.float32, 1)
    if row_index is not None:
        _need_cuda("row_index", row_index, torch.int32, 1)
    _need_cuda("expert_offsets", expert_offsets, torch.int64, 1)
    dev = q_x.device
    E = expert_offsets.numel() - 1
    T, K = q_x.shape
    R = row_index.numel() if row_index is not None else T
    if isinstance(packed, torch.Tensor):
        wp = packed
    else:
        if len(packed) != E or len(S) != E:
            raise ValueError("one packed weight and one integer-scale tensor per expert")
        if N is None:
            N = int(next((t.shape[0] for t in packed if t is not None), 0))
        wp = device_pointers(packed, dev)
    sp = S if isinstance(S, torch.Tensor) else device_pointers(S, dev)
    _need_cuda("packed pointers", wp, torch.int64, 1)
    _need_cuda("S pointers", sp, torch.int64, 1)
    if N is None:
        raise ValueError("N must be given with pointer arrays")
    if out_row is not None:
        _need_cuda("out_row", out_row, torch.int32, 1)
    dt, tdt = _OUT[out]
    if y is None:
        rows = R if out_row is None else (int(y_rows) if y_rows is not None else R)
        y = torch.empty((rows, N), dtype=tdt, device=dev)
    _need_cuda("y", y, tdt, 2)
    if workspace is None:
        workspace = grouped_workspace(E, N, K, group, dev)
    code = load().w4a8_gemm_intscale_grouped(_ptr(q_x), _ptr(s_a), T, _ptr(row_index), _ptr(expert_offsets),
                                             _ptr(out_row), _ptr(wp), _ptr(sp), int(alpha), E, R, N, K, group,
                                             _ptr(y), dt, y.shape[0], _ptr(workspace), workspace.numel(),
                                             _stream(dev))
    _check("w4a8_gemm_intscale_grouped", code)
    return y


def tensor_i8_peak_probe(iters: int, n: int = 256, a_in_tmem: bool = False, device=None) -> float:
    """Launch the int8 tensor-pipe probe on the current stream of `device`
    (back-to-back 128 x n x 32 MMAs on on-chip operands, one CTA per SM) and
    return the int8 operations it performs; time it with CUDA events."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    grid = ctypes.c_int32(0)
    ops = ctypes.c_double(0.0)
    with torch.cuda.device(device):
        code = load().w4a8_tensor_i8_peak_probe(int(iters), int(n), 1 if a_in_tmem else 0, ctypes.byref(grid),
                                                ctypes.byref(ops), _stream(device))
    _check("w4a8_tensor_i8_peak_probe", code)
    return float(ops.value)


def device_status(clear: bool = True) -> int:
    """The device status word (0, or the code of a kernel wait that timed
    out); a nonzero status also re-zeroes the cached GEMM workspaces."""
    v = ctypes.c_int32(0)
    _check("w4a8_device_status", load().w4a8_device_status(ctypes.byref(v), 1 if clear else 0))
    if v.value != 0:
        _reset_workspaces()
    return int(v.value)
