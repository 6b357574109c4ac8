"""Tensor-parallel reconciliation point on one B200 (sm_100a).

A row-parallel projection split across N ranks: each rank's partial x_r . W_r,
summed in ring all-reduce order (reduce-scatter then all-gather of H/N
chunks, bf16 round-to-nearest-even after each add), then the residual add.
All N ranks are emulated in one GPU's memory. The computation lives in
``libtp_reconcile.so`` (hand-written CUDA for sm_100a, C ABI in
include/tp_reconcile.h); this package only binds it.
"""

from ._lib import (EXPORTED, LIB_PATH, TP_BF16, TP_ERR_ALIGN, TP_ERR_CUDA, TP_ERR_INVALID,
                   TP_ERR_UNSUPPORTED, TP_ERR_WORKSPACE, TP_OK, TP_VARIANT_AUTO, TP_VARIANT_CLUSTER, TP_VARIANT_EXACT,
                   TP_VARIANT_TENSOR, TPError, tp_device_error_flags, tp_last_cuda_error,
                   tp_pack_weights, tp_plan_create, tp_plan_destroy, tp_plan_set_variant,
                   tp_allreduce_bytes, tp_moe_combine_bytes, tp_pack_weights_mxfp8,
                   tp_ring_rank_workspace_bytes, tp_ring_allreduce_ranks, tp_plan_mxfp8_bytes,
                   tp_rowlinear_reconcile_mxfp8, tp_plan_mxfp8_workspace_bytes, TP_ALLREDUCE_NAIVE,
                   tp_plan_nvfp4_bytes, tp_pack_weights_nvfp4, tp_plan_nvfp4_workspace_bytes,
                   tp_rowlinear_reconcile_nvfp4, TP_ALLREDUCE_RING,
                   TP_ALLREDUCE_SWITCH, tp_plan_kernel_variant, tp_plan_launches, tp_plan_packed_bytes, tp_plan_workspace_bytes, tp_ring_bytes, tp_ring_reduce, tp_rowlinear_partials,
                   tp_rowlinear_reconcile, tp_rowlinear_reconcile_noalloc, tp_status_string)
from .plan import Plan, ring_bytes

__all__ = [
    "Plan", "ring_bytes", "TPError", "LIB_PATH", "EXPORTED",
    "tp_plan_create", "tp_plan_set_variant", "tp_plan_workspace_bytes", "tp_plan_kernel_variant",
    "tp_plan_launches", "tp_plan_packed_bytes", "tp_pack_weights",
    "tp_rowlinear_reconcile", "tp_rowlinear_reconcile_noalloc", "tp_rowlinear_partials",
    "tp_ring_reduce", "tp_ring_bytes", "tp_allreduce_bytes", "tp_moe_combine_bytes",
    "tp_ring_rank_workspace_bytes", "tp_ring_allreduce_ranks",
    "TP_ALLREDUCE_RING", "TP_ALLREDUCE_NAIVE", "TP_ALLREDUCE_SWITCH",
    "tp_plan_mxfp8_bytes", "tp_pack_weights_mxfp8", "tp_plan_mxfp8_workspace_bytes",
    "tp_rowlinear_reconcile_mxfp8", "tp_plan_nvfp4_bytes", "tp_pack_weights_nvfp4",
    "tp_plan_nvfp4_workspace_bytes", "tp_rowlinear_reconcile_nvfp4",
    "tp_plan_destroy", "tp_status_string", "tp_last_cuda_error", "tp_device_error_flags",
    "TP_OK", "TP_ERR_INVALID", "TP_ERR_ALIGN", "TP_ERR_UNSUPPORTED", "TP_ERR_WORKSPACE",
    "TP_ERR_CUDA", "TP_BF16", "TP_VARIANT_AUTO", "TP_VARIANT_EXACT", "TP_VARIANT_TENSOR", "TP_VARIANT_CLUSTER",
]
