"""Torch-facing wrapper of the C ABI: a ``Plan`` owns one tp_plan handle.

PyTorch supplies device memory and the current stream; every tensor goes to
the library as a data pointer after its device, dtype, shape and layout are
checked here. Nothing is computed in Python.
"""

from __future__ import annotations

from typing import Optional

import torch

from . import _lib
from ._lib import TPError

_VARIANTS = {"auto": _lib.TP_VARIANT_AUTO, "exact": _lib.TP_VARIANT_EXACT,
             "tensor": _lib.TP_VARIANT_TENSOR, "cluster": _lib.TP_VARIANT_CLUSTER}


def _check(t: torch.Tensor, name: str, shape) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


class Plan:
    """One projection shape: N ranks, up to max_tokens tokens, K inputs, H outputs."""

    def __init__(self, n_ranks: int, max_tokens: int, k: int, hidden: int,
                 variant: str = "auto", staged: bool = False):
        st, h = _lib.tp_plan_create(n_ranks, max_tokens, k, hidden, _lib.TP_BF16)
        if st != _lib.TP_OK:
            raise TPError(st, "tp_plan_create")
        self._h = h
        self.n_ranks, self.max_tokens, self.k, self.hidden = n_ranks, max_tokens, k, hidden
        self.ks, self.hc = k // n_ranks, hidden // n_ranks
        self.device = torch.cuda.current_device()
        self.set_variant(variant, staged)

    def set_variant(self, variant: str = "auto", staged: bool = False) -> None:
        st = _lib.tp_plan_set_variant(self._h, _VARIANTS[variant], int(bool(staged)))
        if st != _lib.TP_OK:
            raise TPError(st, "tp_plan_set_variant")
        self.variant, self.staged = variant, bool(staged)

    @property
    def handle(self):
        return self._h

    def close(self) -> None:
        if getattr(self, "_h", None):
            _lib.tp_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace_bytes(self, tokens: int) -> int:
        return _lib.tp_plan_workspace_bytes(self._h, tokens)

    def effective_variant(self, tokens: int) -> str:
        """'exact' or 'tensor': the partial kernel a call with this many tokens runs."""
        v = _lib.tp_plan_kernel_variant(self._h, tokens)
        if v < 0:
            raise ValueError("tokens must be >= 1")
        return "tensor" if v == _lib.TP_VARIANT_TENSOR else "exact"

    def launches(self, tokens: int) -> int:
        """Kernels one reconcile call with this many tokens launches."""
        return _lib.tp_plan_launches(self._h, tokens)

    @property
    def packed_numel(self) -> int:
        """bf16 elements of the packed weight buffer (tiled shards, see tp_reconcile.h)."""
        return _lib.tp_plan_packed_bytes(self._h) // 2

    def pack_weights(self, w_hk: torch.Tensor, out: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
        """Linear weight [H, K] -> packed tiled shards (flat bf16 tensor)."""
        if out is None:
            out = torch.empty(self.packed_numel, dtype=torch.bfloat16, device=w_hk.device)
        a = _check(w_hk, "w_hk", (self.hidden, self.k))
        b = _check(out, "w_packed", (self.packed_numel,))
        st = _lib.tp_pack_weights(self._h, a, b, _stream(stream))
        if st != _lib.TP_OK:
            raise TPError(st, "tp_pack_weights")
        return out

    def reconcile(self, x: torch.Tensor, w_packed: torch.Tensor, residual: torch.Tensor,
                  out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  stream=None) -> torch.Tensor:
        """out [M, H] = residual + ring-ordered sum over ranks of x_r . W_r^T."""
        m = x.shape[0]
        if out is None:
            out = torch.empty(m, self.hidden, dtype=torch.bfloat16, device=x.device)
        px = _check(x, "x", (m, self.k))
        pw = _check(w_packed, "w_packed", (self.packed_numel,))
        pr = _check(residual, "residual", (m, self.hidden))
        po = _check(out, "out", (m, self.hidden))
        need = self.workspace_bytes(m)
        pws = 0
        if need:
            if workspace is None:   # fold counters start at zero
                workspace = torch.zeros(need, dtype=torch.uint8, device=x.device)
            if workspace.numel() * workspace.element_size() < need or workspace.device.type != "cuda":
                raise ValueError("workspace too small")
            pws = workspace.data_ptr()
        st = _lib.tp_rowlinear_reconcile(self._h, px, pw, pr, po, m, pws, _stream(stream))
        if st != _lib.TP_OK:
            raise TPError(st, "tp_rowlinear_reconcile")
        return out

    # ---------------------------------------------------- MXFP8 shards --

    def mxfp8_bytes(self):
        """(code bytes, scale bytes) of this plan's MXFP8 shards."""
        st, q, sc = _lib.tp_plan_mxfp8_bytes(self._h)
        if st != _lib.TP_OK:
            raise TPError(st, "tp_plan_mxfp8_bytes")
        return q, sc

    def pack_weights_mxfp8(self, w_hk: torch.Tensor, stream=None):
        """Linear weight [H, K] -> (E4M3 codes, E8M0 scales) as flat uint8 tensors."""
        qb, sb = self.mxfp8_bytes()
        q = torch.empty(qb, dtype=torch.uint8, device=w_hk.device)
        sc = torch.empty(sb, dtype=torch.uint8, device=w_hk.device)
        a = _check(w_hk, "w_hk", (self.hidden, self.k))
        st = _lib.tp_pack_weights_mxfp8(self._h, a, q.data_ptr(), sc.data_ptr(), _stream(stream))
        if st != _lib.TP_OK:
            raise TPError(st, "tp_pack_weights_mxfp8")
        return q, sc

    def mxfp8_workspace_bytes(self, tokens: int) -> int:
        return _lib.tp_plan_mxfp8_workspace_bytes(self._h, tokens)

    def reconcile_mxfp8(self, x: torch.Tensor, w_q: torch.Tensor, w_scales: torch.Tensor,
                        residual: torch.Tensor, out: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """out [M, H] = residual + ring-ordered sum of x_r . dequant(W_r)^T."""
        m = x.shape[0]
        if out is None:
            out = torch.empty(m, self.hidden, dtype=torch.bfloat16, device=x.device)
        qb, sb = self.mxfp8_bytes()
        for t, name, n in ((w_q, "w_q", qb), (w_scales, "w_scales", sb)):
            if t.dtype != torch.uint8 or t.numel() != n or t.device.type != "cuda" or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous CUDA uint8 tensor of {n} bytes")
        px = _check(x, "x", (m, self.k))
        pr = _check(residual, "residual", (m, self.hidden))
        po = _check(out, "out", (m, self.hidden))
        need = self.mxfp8_workspace_bytes(m)
        pws = 0
        if need:
            if workspace is None:   # fold counters start at zero
                workspace = torch.zeros(need, dtype=torch.uint8, device=x.device)
            if workspace.numel() * workspace.element_size() < need or workspace.device.type != "cuda":
                raise ValueError("workspace too small")
            pws = workspace.data_ptr()
        st = _lib.tp_rowlinear_reconcile_mxfp8(self._h, px, w_q.data_ptr(), w_scales.data_ptr(), pr, po,
                                               m, pws, _stream(stream))
        if st != _lib.TP_OK:
            raise TPError(st, "tp_rowlinear_reconcile_mxfp8")
        return out

    # ---------------------------------------------------- NVFP4 shards --

    def nvfp4_bytes(self):
        """(code bytes, scale bytes) of this plan's NVFP4 shards."""
        st, q, sc = _lib.tp_plan_nvfp4_bytes(self._h)
        if st != _lib.TP_OK:
            raise TPError(st, "tp_plan_nvfp4_bytes")
        return q, sc

    def nvfp4_workspace_bytes(self, tokens: int) -> int:
        return _lib.tp_plan_nvfp4_workspace_bytes(self._h, tokens)

    def pack_weights_nvfp4(self, w_hk: torch.Tensor, stream=None):
        """Linear weight [H, K] -> (E2M1 code pairs, E4M3 block scales + g) as flat uint8 tensors."""
        qb, sb = self.nvfp4_bytes()
        q = torch.empty(qb, dtype=torch.uint8, device=w_hk.device)
        sc = torch.empty(sb, dtype=torch.uint8, device=w_hk.device)
        a = _check(w_hk, "w_hk", (self.hidden, self.k))
        st = _lib.tp_pack_weights_nvfp4(self._h, a, q.data_ptr(), sc.data_ptr(), _stream(stream))
        if st != _lib.TP_OK:
            raise TPError(st, "tp_pack_weights_nvfp4")
        return q, sc

    def reconcile_nvfp4(self, x: torch.Tensor, w_q: torch.Tensor, w_scales: torch.Tensor,
                        residual: torch.Tensor, out: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """out [M, H] = residual + ring-ordered sum of x_r . dequant(W_r)^T (NVFP4 shards)."""
        m = x.shape[0]
        if out is None:
            out = torch.empty(m, self.hidden, dtype=torch.bfloat16, device=x.device)
        qb, sb = self.nvfp4_bytes()
        for t, name, n in ((w_q, "w_q", qb), (w_scales, "w_scales", sb)):
            if t.dtype != torch.uint8 or t.numel() != n or t.device.type != "cuda" or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous CUDA uint8 tensor of {n} bytes")
        px = _check(x, "x", (m, self.k))
        pr = _check(residual, "residual", (m, self.hidden))
        po = _check(out, "out", (m, self.hidden))
        need = self.nvfp4_workspace_bytes(m)
        pws = 0
        if need:
            if workspace is None:   # fold counters start at zero
                workspace = torch.zeros(need, dtype=torch.uint8, device=x.device)
            if workspace.numel() * workspace.element_size() < need or workspace.device.type != "cuda":
                raise ValueError("workspace too small")
            pws = workspace.data_ptr()
        st = _lib.tp_rowlinear_reconcile_nvfp4(self._h, px, w_q.data_ptr(), w_scales.data_ptr(), pr, po,
                                               m, pws, _stream(stream))
        if st != _lib.TP_OK:
            raise TPError(st, "tp_rowlinear_reconcile_nvfp4")
        return out

    def partials(self, x: torch.Tensor, w_packed: torch.Tensor,
                 out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """The N partials [N, M, H] (S1 only)."""
        m = x.shape[0]
        if out is None:
            out = torch.empty(self.n_ranks, m, self.hidden, dtype=torch.bfloat16, device=x.device)
        px = _check(x, "x", (m, self.k))
        pw = _check(w_packed, "w_packed", (self.packed_numel,))
        po = _check(out, "partials", (self.n_ranks, m, self.hidden))
        st = _lib.tp_rowlinear_partials(self._h, px, pw, po, m, _stream(stream))
        if st != _lib.TP_OK:
            raise TPError(st, "tp_rowlinear_partials")
        return out

    def ring_reduce(self, partials: torch.Tensor, residual: torch.Tensor,
                    out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """S2-S4 on given partials [N, M, H]."""
        m = partials.shape[1]
        if out is None:
            out = torch.empty(m, self.hidden, dtype=torch.bfloat16, device=partials.device)
        pp = _check(partials, "partials", (self.n_ranks, m, self.hidden))
        pr = _check(residual, "residual", (m, self.hidden))
        po = _check(out, "out", (m, self.hidden))
        st = _lib.tp_ring_reduce(self._h, pp, pr, po, m, _stream(stream))
        if st != _lib.TP_OK:
            raise TPError(st, "tp_ring_reduce")
        return out

    def ring_rank_workspace_bytes(self, tokens: int) -> int:
        return _lib.tp_ring_rank_workspace_bytes(self._h, tokens)

    def ring_allreduce_ranks(self, partials, residual: torch.Tensor, outs=None, workspaces=None,
                             first_rank: int = 0, launch_ranks: Optional[int] = None,
                             wait_limit_ns: int = 0, stream=None):
        """The ring all-reduce as a protocol between ranks with their own
        buffers: partials and outs are N tensors [M, H] (one per rank),
        workspaces N uint8 tensors of ring_rank_workspace_bytes (zeroed when
        created here). Runs ranks first_rank .. first_rank + launch_ranks - 1
        (default: all). Returns (outs, workspaces)."""
        n = self.n_ranks
        if len(partials) != n:
            raise ValueError(f"need {n} partials")
        m = partials[0].shape[0]
        pp = [_check(t, f"partials[{i}]", (m, self.hidden)) for i, t in enumerate(partials)]
        pr = _check(residual, "residual", (m, self.hidden))
        if outs is None:
            outs = [torch.empty(m, self.hidden, dtype=torch.bfloat16, device=residual.device)
                    for _ in range(n)]
        po = [_check(t, f"outs[{i}]", (m, self.hidden)) for i, t in enumerate(outs)]
        need = self.ring_rank_workspace_bytes(m)
        if workspaces is None:
            workspaces = [torch.zeros(need, dtype=torch.uint8, device=residual.device) for _ in range(n)]
        for i, w in enumerate(workspaces):
            if w.device.type != "cuda" or w.numel() * w.element_size() < need:
                raise ValueError(f"workspaces[{i}] too small")
        st = _lib.tp_ring_allreduce_ranks(self._h, pp, pr, po, [w.data_ptr() for w in workspaces],
                                          first_rank, n if launch_ranks is None else launch_ranks, m,
                                          wait_limit_ns, _stream(stream))
        if st != _lib.TP_OK:
            raise TPError(st, "tp_ring_allreduce_ranks")
        return outs, workspaces

    def device_error_flags(self, reset: bool = False) -> int:
        st, flags = _lib.tp_device_error_flags(self._h, int(reset))
        if st != _lib.TP_OK:
            raise TPError(st, "tp_device_error_flags")
        return flags


def ring_bytes(n_ranks: int, tokens: int, hidden: int, elem_bytes: int = 2, points: int = 1) -> int:
    return _lib.tp_ring_bytes(n_ranks, tokens, hidden, elem_bytes, points)
