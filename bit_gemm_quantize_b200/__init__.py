"""W4A8 Integer-Scale linear-layer compute for NVIDIA B200 (sm_100a).

The computation runs in the CUDA library built from ``csrc/`` (C ABI in
``include/w4a8_intscale.h``); this package is its Python binding plus the
seeded synthetic workload generator used by the tests and the benchmark.
"""
from ._native import (  # noqa: F401
    W4A8Error,
    device_status,
    gemm_workspace,
    load,
    grouped_workspace,
    device_pointers,
    pack_moe_experts,
    pack_w4_groupwise,
    pack_w8_groupwise,
    quantize_act_per_token,
    quantize_act_per_token_asym,
    quantize_act_routed,
    tensor_i8_peak_probe,
    w4_zero_point_term,
    w4a8_amplifier_search,
    w4a8_gemm_floatscale,
    w4a8_gemm_intscale,
    w4a8_gemm_intscale_asym,
    w4a8_gemm_intscale_static_ws,
    w4a8_gemm_intscale_grouped,
    w4a8_linear_intscale,
    w8a8_gemm_intscale,
)

__all__ = [
    "W4A8Error",
    "device_status",
    "gemm_workspace",
    "load",
    "grouped_workspace",
    "device_pointers",
    "pack_moe_experts",
    "pack_w4_groupwise",
    "pack_w8_groupwise",
    "quantize_act_per_token",
    "quantize_act_per_token_asym",
    "quantize_act_routed",
    "tensor_i8_peak_probe",
    "w4_zero_point_term",
    "w4a8_amplifier_search",
    "w4a8_gemm_floatscale",
    "w4a8_gemm_intscale",
    "w4a8_gemm_intscale_asym",
    "w4a8_gemm_intscale_static_ws",
    "w4a8_gemm_intscale_grouped",
    "w4a8_linear_intscale",
    "w8a8_gemm_intscale",
]
