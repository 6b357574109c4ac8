"""ctypes binding of the C ABI in include/tp_reconcile.h (argument marshalling only).

Every function here has the name and argument order of its C counterpart and
passes plain integers (device pointers, sizes, a cudaStream_t) through. All
computation happens in libtp_reconcile.so; if that library is missing or does
not load, importing this module raises -- there is no other code path.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtp_reconcile.so")

TP_OK, TP_ERR_INVALID, TP_ERR_ALIGN, TP_ERR_UNSUPPORTED, TP_ERR_WORKSPACE, TP_ERR_CUDA = range(6)
TP_BF16 = 0
TP_VARIANT_AUTO, TP_VARIANT_EXACT, TP_VARIANT_TENSOR, TP_VARIANT_CLUSTER = 0, 1, 2, 3

EXPORTED = (
    "tp_plan_create", "tp_plan_set_variant", "tp_plan_workspace_bytes", "tp_plan_kernel_variant", "tp_plan_launches",
    "tp_plan_packed_bytes",
    "tp_pack_weights",
    "tp_rowlinear_reconcile", "tp_rowlinear_reconcile_noalloc", "tp_rowlinear_partials",
    "tp_ring_reduce", "tp_ring_bytes", "tp_allreduce_bytes", "tp_moe_combine_bytes",
    "tp_ring_rank_workspace_bytes", "tp_ring_allreduce_ranks",
    "tp_plan_mxfp8_bytes", "tp_pack_weights_mxfp8", "tp_plan_mxfp8_workspace_bytes",
    "tp_rowlinear_reconcile_mxfp8", "tp_plan_nvfp4_bytes", "tp_pack_weights_nvfp4",
    "tp_plan_nvfp4_workspace_bytes", "tp_rowlinear_reconcile_nvfp4",
    "tp_plan_destroy", "tp_status_string", "tp_last_cuda_error", "tp_device_error_flags",
)


class TPError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _status_string(status)
        if status == TP_ERR_CUDA:
            msg += f" (cudaError {LIB.tp_last_cuda_error()})"
        super().__init__(f"{where}: {msg}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with tensor_layer_reconciliation_b200/build.py "
            "(nvcc, sm_100a). There is no fallback implementation.")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
    L.tp_plan_create.argtypes = [ctypes.POINTER(vp), ctypes.c_int, i64, i64, i64, ctypes.c_int]
    L.tp_plan_create.restype = ctypes.c_int
    L.tp_plan_set_variant.argtypes = [vp, ctypes.c_int, ctypes.c_int]
    L.tp_plan_set_variant.restype = ctypes.c_int
    L.tp_plan_workspace_bytes.argtypes = [vp, i64]
    L.tp_plan_workspace_bytes.restype = sz
    L.tp_plan_kernel_variant.argtypes = [vp, i64]
    L.tp_plan_kernel_variant.restype = ctypes.c_int
    L.tp_plan_launches.argtypes = [vp, i64]
    L.tp_plan_launches.restype = ctypes.c_int
    L.tp_plan_packed_bytes.argtypes = [vp]
    L.tp_plan_packed_bytes.restype = sz
    L.tp_pack_weights.argtypes = [vp, vp, vp, vp]
    L.tp_pack_weights.restype = ctypes.c_int
    L.tp_rowlinear_reconcile.argtypes = [vp, vp, vp, vp, vp, i64, vp, vp]
    L.tp_rowlinear_reconcile.restype = ctypes.c_int
    L.tp_rowlinear_reconcile_noalloc.argtypes = [vp, vp, vp, vp, vp, i64, vp]
    L.tp_rowlinear_reconcile_noalloc.restype = ctypes.c_int
    L.tp_rowlinear_partials.argtypes = [vp, vp, vp, vp, i64, vp]
    L.tp_rowlinear_partials.restype = ctypes.c_int
    L.tp_ring_reduce.argtypes = [vp, vp, vp, vp, i64, vp]
    L.tp_ring_reduce.restype = ctypes.c_int
    L.tp_ring_bytes.argtypes = [ctypes.c_int, i64, i64, ctypes.c_int, i64]
    L.tp_ring_bytes.restype = ctypes.c_uint64
    L.tp_plan_mxfp8_bytes.argtypes = [vp, ctypes.POINTER(sz), ctypes.POINTER(sz)]
    L.tp_plan_mxfp8_bytes.restype = ctypes.c_int
    L.tp_pack_weights_mxfp8.argtypes = [vp, vp, vp, vp, vp]
    L.tp_pack_weights_mxfp8.restype = ctypes.c_int
    L.tp_rowlinear_reconcile_mxfp8.argtypes = [vp, vp, vp, vp, vp, vp, i64, vp, vp]
    L.tp_plan_mxfp8_workspace_bytes.argtypes = [vp, i64]
    L.tp_plan_mxfp8_workspace_bytes.restype = sz
    L.tp_plan_nvfp4_bytes.argtypes = [vp, ctypes.POINTER(sz), ctypes.POINTER(sz)]
    L.tp_plan_nvfp4_bytes.restype = ctypes.c_int
    L.tp_pack_weights_nvfp4.argtypes = [vp, vp, vp, vp, vp]
    L.tp_pack_weights_nvfp4.restype = ctypes.c_int
    L.tp_plan_nvfp4_workspace_bytes.argtypes = [vp, i64]
    L.tp_plan_nvfp4_workspace_bytes.restype = sz
    L.tp_rowlinear_reconcile_nvfp4.argtypes = [vp, vp, vp, vp, vp, vp, i64, vp, vp]
    L.tp_rowlinear_reconcile_nvfp4.restype = ctypes.c_int
    L.tp_rowlinear_reconcile_mxfp8.restype = ctypes.c_int
    L.tp_allreduce_bytes.argtypes = [ctypes.c_int, ctypes.c_int, i64, i64, ctypes.c_int, i64]
    L.tp_allreduce_bytes.restype = ctypes.c_uint64
    L.tp_moe_combine_bytes.argtypes = [ctypes.c_int, ctypes.c_int, i64, i64, ctypes.c_int, i64,
                                       ctypes.c_int]
    L.tp_moe_combine_bytes.restype = ctypes.c_uint64
    L.tp_ring_rank_workspace_bytes.argtypes = [vp, i64]
    L.tp_ring_rank_workspace_bytes.restype = sz
    vpp = ctypes.POINTER(ctypes.c_void_p)
    L.tp_ring_allreduce_ranks.argtypes = [vp, vpp, vp, vpp, vpp, ctypes.c_int, ctypes.c_int, i64,
                                          ctypes.c_uint64, vp]
    L.tp_ring_allreduce_ranks.restype = ctypes.c_int
    L.tp_plan_destroy.argtypes = [vp]
    L.tp_plan_destroy.restype = None
    L.tp_status_string.argtypes = [ctypes.c_int]
    L.tp_status_string.restype = ctypes.c_char_p
    L.tp_last_cuda_error.argtypes = []
    L.tp_last_cuda_error.restype = ctypes.c_int
    L.tp_device_error_flags.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32), ctypes.c_int]
    L.tp_device_error_flags.restype = ctypes.c_int
    return L


LIB = _load()


def _status_string(status: int) -> str:
    return LIB.tp_status_string(status).decode()


# ---- the C ABI, name for name --------------------------------------------

def tp_plan_create(n_ranks: int, max_tokens: int, k: int, hidden: int, dtype: int = TP_BF16):
    """Returns (status, plan handle or None)."""
    h = ctypes.c_void_p()
    st = LIB.tp_plan_create(ctypes.byref(h), n_ranks, max_tokens, k, hidden, dtype)
    return st, (h.value if st == TP_OK else None)


def tp_plan_set_variant(plan, variant: int, staged: int) -> int:
    return LIB.tp_plan_set_variant(plan, variant, staged)


def tp_plan_workspace_bytes(plan, tokens: int) -> int:
    return LIB.tp_plan_workspace_bytes(plan, tokens)


def tp_plan_kernel_variant(plan, tokens: int) -> int:
    return LIB.tp_plan_kernel_variant(plan, tokens)


def tp_plan_launches(plan, tokens: int) -> int:
    return LIB.tp_plan_launches(plan, tokens)


def tp_plan_packed_bytes(plan) -> int:
    return LIB.tp_plan_packed_bytes(plan)


def tp_pack_weights(plan, w_hk: int, w_packed: int, stream: int) -> int:
    return LIB.tp_pack_weights(plan, w_hk, w_packed, stream)


def tp_rowlinear_reconcile(plan, x: int, w_packed: int, residual: int, out: int, tokens: int,
                           workspace: int, stream: int) -> int:
    return LIB.tp_rowlinear_reconcile(plan, x, w_packed, residual, out, tokens, workspace, stream)


def tp_rowlinear_reconcile_noalloc(plan, x: int, w_packed: int, residual: int, out: int,
                                   tokens: int, stream: int) -> int:
    """tp_rowlinear_reconcile with the library's fixed scratch instead of a workspace."""
    return LIB.tp_rowlinear_reconcile_noalloc(plan, x, w_packed, residual, out, tokens, stream)


def tp_rowlinear_partials(plan, x: int, w_packed: int, partials: int, tokens: int,
                          stream: int) -> int:
    return LIB.tp_rowlinear_partials(plan, x, w_packed, partials, tokens, stream)


def tp_ring_reduce(plan, partials: int, residual: int, out: int, tokens: int, stream: int) -> int:
    return LIB.tp_ring_reduce(plan, partials, residual, out, tokens, stream)


def tp_plan_mxfp8_bytes(plan):
    q, sc = ctypes.c_size_t(0), ctypes.c_size_t(0)
    st = LIB.tp_plan_mxfp8_bytes(plan, ctypes.byref(q), ctypes.byref(sc))
    return st, q.value, sc.value


def tp_pack_weights_mxfp8(plan, w_hk: int, w_q: int, w_scales: int, stream: int) -> int:
    return LIB.tp_pack_weights_mxfp8(plan, w_hk, w_q, w_scales, stream)


def tp_rowlinear_reconcile_mxfp8(plan, x: int, w_q: int, w_scales: int, residual: int, out: int,
                                 tokens: int, workspace: int, stream: int) -> int:
    return LIB.tp_rowlinear_reconcile_mxfp8(plan, x, w_q, w_scales, residual, out, tokens, workspace,
                                            stream)


def tp_plan_mxfp8_workspace_bytes(plan, tokens: int) -> int:
    return LIB.tp_plan_mxfp8_workspace_bytes(plan, tokens)


def tp_plan_nvfp4_bytes(plan):
    q, sc = ctypes.c_size_t(0), ctypes.c_size_t(0)
    st = LIB.tp_plan_nvfp4_bytes(plan, ctypes.byref(q), ctypes.byref(sc))
    return st, q.value, sc.value


def tp_pack_weights_nvfp4(plan, w_hk: int, w_q: int, w_scales: int, stream: int) -> int:
    return LIB.tp_pack_weights_nvfp4(plan, w_hk, w_q, w_scales, stream)


def tp_plan_nvfp4_workspace_bytes(plan, tokens: int) -> int:
    return LIB.tp_plan_nvfp4_workspace_bytes(plan, tokens)


def tp_rowlinear_reconcile_nvfp4(plan, x: int, w_q: int, w_scales: int, residual: int, out: int,
                                 tokens: int, workspace: int, stream: int) -> int:
    return LIB.tp_rowlinear_reconcile_nvfp4(plan, x, w_q, w_scales, residual, out, tokens, workspace,
                                            stream)


TP_ALLREDUCE_RING, TP_ALLREDUCE_NAIVE, TP_ALLREDUCE_SWITCH = 0, 1, 2


def tp_allreduce_bytes(scheme: int, n_ranks: int, tokens: int, hidden: int, elem_bytes: int,
                       points: int) -> int:
    return int(LIB.tp_allreduce_bytes(scheme, n_ranks, tokens, hidden, elem_bytes, points))


def tp_moe_combine_bytes(scheme: int, n_ranks: int, tokens: int, hidden: int, elem_bytes: int,
                         top_k: int, local_accumulate: int = 1) -> int:
    return int(LIB.tp_moe_combine_bytes(scheme, n_ranks, tokens, hidden, elem_bytes, top_k,
                                        local_accumulate))


def tp_ring_rank_workspace_bytes(plan, tokens: int) -> int:
    return LIB.tp_ring_rank_workspace_bytes(plan, tokens)


def tp_ring_allreduce_ranks(plan, partials, residual: int, outs, workspaces, first_rank: int,
                            launch_ranks: int, tokens: int, wait_limit_ns: int, stream: int) -> int:
    """partials, outs, workspaces: sequences of N device addresses (or None)."""
    def arr(ptrs):
        if ptrs is None:
            return None
        a = (ctypes.c_void_p * len(ptrs))(*[ctypes.c_void_p(int(v) if v else None) for v in ptrs])
        return ctypes.cast(a, ctypes.POINTER(ctypes.c_void_p))
    return LIB.tp_ring_allreduce_ranks(plan, arr(partials), residual, arr(outs), arr(workspaces),
                                       first_rank, launch_ranks, tokens, wait_limit_ns, stream)


def tp_ring_bytes(n_ranks: int, tokens: int, hidden: int, elem_bytes: int, points: int) -> int:
    return int(LIB.tp_ring_bytes(n_ranks, tokens, hidden, elem_bytes, points))


def tp_plan_destroy(plan) -> None:
    LIB.tp_plan_destroy(plan)


def tp_status_string(status: int) -> str:
    return _status_string(status)


def tp_last_cuda_error() -> int:
    return LIB.tp_last_cuda_error()


def tp_device_error_flags(plan, reset: int = 0):
    """Returns (status, flags)."""
    v = ctypes.c_uint32(0)
    st = LIB.tp_device_error_flags(plan, ctypes.byref(v), reset)
    return st, v.value
