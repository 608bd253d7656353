"""B200-native MoE expert-parallel token dispatch and combine.

The work runs in libep.so (C ABI in include/ep.h, sm_100a CUDA kernels);
``ep`` is its thin Python binding.  Importing the package without the built
library raises ImportError: there is no CPU or library fallback.
"""
from .ep import (GROUP_KIND_BACKWARD, GROUP_KIND_COMBINED, GROUP_KIND_COUNTS, GROUP_KIND_DISPATCH,
                 GROUP_KIND_EXPERT_OUT, GROUP_KINDS, EpGroupT, EpPeers, ep_group_combine,
                 ep_group_combine_backward, ep_group_dispatch, ep_group_layout, ep_group_plan,
                 ep_group_plan_host, ep_group_signal, ep_group_sizes, ep_group_wait, ep_ipc_close,
                 ep_ipc_export, ep_ipc_import, make_group,
                 DEV_BAD_INDEX, DEV_CAPACITY_OVERFLOW, DEV_TIMEOUT, ERR_BUFFER_TOO_SMALL,
                 STATIC_SCRATCH_BYTES, F_BWD_UNWEIGHTED,
                 F_COMBINE_QUANTIZED, F_GEMM_CTA_PAIRS, F_IDX_I32, F_LAYOUT_CLUSTER, F_LAYOUT_MULTI_CTA,
                 F_LAYOUT_SINGLE_CTA, F_ROUND_SCALE, F_UE8M0, LAYOUT, QUANT, Bound, Buffers,
                 EpConfig, EpError, EpSizes, ep_buffer_sizes, ep_combine, ep_combine_backward,
                 ep_combine_backward_weights, ep_copy, ep_cvt_sweep, ep_dispatch, ep_dispatch_layout,
                 ep_dispatch_layout_static, ep_dispatch_with_layout, ep_expert_ffn_mx, ep_expert_gemm, ep_expert_gemm_mx,
                 ep_ffn_buffer_bytes, ep_moe_forward_ffn,
                 ep_get_status,
                 ep_kernel_launches, ep_moe_forward, ep_wait_probe, idx_dtype,
                 make_config)

__all__ = [
    "GROUP_KIND_BACKWARD", "GROUP_KIND_COMBINED", "GROUP_KIND_COUNTS", "GROUP_KIND_DISPATCH",
    "GROUP_KIND_EXPERT_OUT",
    "GROUP_KINDS", "EpGroupT", "EpPeers", "ep_group_combine", "ep_group_combine_backward",
    "ep_group_dispatch", "ep_group_layout", "ep_group_plan", "ep_group_plan_host",
    "ep_group_signal", "ep_group_sizes", "ep_group_wait", "ep_ipc_close", "ep_ipc_export",
    "ep_ipc_import", "make_group",
    "DEV_BAD_INDEX", "DEV_CAPACITY_OVERFLOW", "DEV_TIMEOUT", "ERR_BUFFER_TOO_SMALL",
    "STATIC_SCRATCH_BYTES", "F_BWD_UNWEIGHTED",
    "F_COMBINE_QUANTIZED", "F_GEMM_CTA_PAIRS", "F_IDX_I32", "F_LAYOUT_CLUSTER", "F_LAYOUT_MULTI_CTA",
    "F_LAYOUT_SINGLE_CTA", "F_ROUND_SCALE", "F_UE8M0", "LAYOUT", "QUANT", "Bound", "Buffers",
    "EpConfig", "EpError", "EpSizes", "ep_buffer_sizes", "ep_combine", "ep_combine_backward",
    "ep_combine_backward_weights",
    "ep_copy", "ep_cvt_sweep", "ep_dispatch", "ep_dispatch_layout", "ep_dispatch_layout_static",
    "ep_dispatch_with_layout", "ep_expert_ffn_mx", "ep_ffn_buffer_bytes", "ep_moe_forward_ffn",
    "ep_expert_gemm", "ep_expert_gemm_mx", "ep_get_status", "ep_kernel_launches", "ep_moe_forward", "ep_wait_probe", "idx_dtype", "make_config",
]
