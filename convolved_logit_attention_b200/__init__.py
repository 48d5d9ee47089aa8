"""Multi-Token Attention (MTA) forward for NVIDIA B200 (sm_100a).

The computation lives in libmta.so (hand-written CUDA, C ABI in
include/mta.h); this package is its Python binding, with the same function
names as the C entry points, plus the seeded synthetic workloads used by the
tests and the benchmark (``convolved_logit_attention_b200.workloads``).
"""
from ._binding import (EXPORTS, LIB_PATH, MTA_BF16, MTA_F32, MTA_PATH_FUSED_TC, MTA_PATH_FUSED_F32,
                       MTA_PATH_MATERIALISED, MtaComposition, MtaError, MtaShape, lib,
                       make_shape, composed_shape, composition, mta_composed_kernel_names,
                       mta_debug_attention, mta_forward_composed, mta_forward, mta_forward_gated, mta_forward_path,
                       mta_forward_traced,
                       mta_forward_unfused, mta_kernel_count, mta_kernel_name,
                       mta_selftest_wait_timeout,
                       mta_status_string, mta_sync_status, mta_unfused_workspace_size,
                       mta_version, mta_workspace_size, shape_of, GRAD_NAMES, mta_backward,
                       mta_backward_kernel_names, mta_backward_workspace_size)

__all__ = ["EXPORTS", "LIB_PATH", "MTA_BF16", "MTA_F32", "MTA_PATH_FUSED_TC", "MTA_PATH_FUSED_F32",
           "MTA_PATH_MATERIALISED", "MtaComposition", "MtaError", "MtaShape", "lib",
           "make_shape", "composed_shape", "composition", "mta_composed_kernel_names",
           "mta_debug_attention", "mta_forward_composed", "mta_forward", "mta_forward_gated", "mta_forward_path",
           "mta_forward_traced",
           "mta_forward_unfused", "mta_kernel_count", "mta_kernel_name",
           "mta_selftest_wait_timeout",
           "mta_status_string", "mta_sync_status", "mta_unfused_workspace_size", "mta_version",
           "mta_workspace_size", "shape_of", "GRAD_NAMES", "mta_backward",
           "mta_backward_kernel_names", "mta_backward_workspace_size"]
