"""PyTorch-facing calls of the draft passes' soft cross-entropy distillation loss.

Argument marshalling only: tensors are checked for dtype, shape, device and
contiguity, outputs and the workspace are allocated with torch, and the C ABI of
libttt_attn.so (``ttt_softce_fwd`` / ``ttt_softce_bwd``) is called on the current CUDA
stream.  Every arithmetic step runs in the library's kernels.

Shapes: h [P, T, d] bf16 (pass-major draft hidden states of the packed tokens), W [V, d]
bf16 (the vocabulary head), y [T, V] bf16 (the teacher's logits), loss_mask [T] uint8
(teacher positions counted), cu_seqlens int32 [nseq + 1] or None (one sequence),
pass_weight / pass_count float32 [P] or None.  Pass p at token t learns the teacher
row t + p of its own sequence.

General form (``row_teacher`` given: e.g. the slots of block drafters, normalised per
slot): row r of h viewed as [P*T, d] learns teacher row row_teacher[r] (int32, -1 =
none) of y [Ty, V] and is normalised in group row_group[r] (int32, None = group 0) of
``ngroups``; loss_mask is [Ty], pass_weight / pass_count [ngroups], the loss [ngroups + 1].
"""

from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def make_desc(h, W, y, cu_seqlens=None, loss_mask=None, pass_weight=None, pass_count=None,
              token_chunk_size: int = 0, events=None, row_teacher=None, row_group=None,
              ngroups: int = 1) -> _lib.TTTSoftceDesc:
    if h.dim() != 3 or W.dim() != 2 or y.dim() != 2:
        raise ValueError("h must be [P, T, d], W [V, d], y [T, V] (or [Ty, V] with row_teacher)")
    P, T, d = h.shape
    V = W.shape[0]
    Ty = y.shape[0] if row_teacher is not None else T
    if W.shape[1] != d or tuple(y.shape) != (Ty, V):
        raise ValueError(f"shape mismatch: h {tuple(h.shape)}, W {tuple(W.shape)}, y {tuple(y.shape)}")
    G = int(ngroups) if row_teacher is not None else int(P)
    for name, t in (("h", h), ("W", W), ("y", y)):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 tensor")
    desc = _lib.TTTSoftceDesc()
    desc.P, desc.T, desc.d, desc.V = int(P), int(T), int(d), int(V)
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be int32 [nseq + 1]")
        desc.cu_seqlens = cu_seqlens.data_ptr()
        desc.nseq = int(cu_seqlens.numel()) - 1
    else:
        desc.cu_seqlens = None
        desc.nseq = 1
    if loss_mask is not None:
        if loss_mask.dtype != torch.uint8 or tuple(loss_mask.shape) != (Ty,):
            raise ValueError("loss_mask must be uint8 [T] ([Ty] with row_teacher)")
        desc.loss_mask = loss_mask.data_ptr()
    for name, t in (("pass_weight", pass_weight), ("pass_count", pass_count)):
        if t is not None:
            if t.dtype != torch.float32 or tuple(t.shape) != (G,):
                raise ValueError(f"{name} must be float32 [P] ([ngroups] with row_teacher)")
            setattr(desc, name, t.data_ptr())
    desc.token_chunk_size = int(token_chunk_size)
    desc.events = ctypes.addressof(events) if events is not None else None
    if row_teacher is not None:
        for name, t in (("row_teacher", row_teacher), ("row_group", row_group)):
            if t is not None and (t.dtype != torch.int32 or tuple(t.shape) != (P * T,) or not t.is_contiguous()):
                raise ValueError(f"{name} must be a contiguous int32 [P*T]")
        desc.row_teacher = row_teacher.data_ptr()
        desc.row_group = None if row_group is None else row_group.data_ptr()
        desc.ngroups = G
        desc.teacher_rows = int(Ty)
    return desc


def ngroups_of(desc: _lib.TTTSoftceDesc) -> int:
    """Normalisation groups of a descriptor: the passes, or ngroups in the general form."""
    return int(desc.ngroups) if desc.row_teacher else int(desc.P)


def workspace_bytes(desc: _lib.TTTSoftceDesc, for_backward) -> int:
    """Workspace of the forward (0 / False), the backward (1 / True) or the fused call (2)."""
    n = _lib.lib().ttt_softce_workspace_size(ctypes.byref(desc), int(for_backward))
    if n == 0:
        raise _lib.TTTError(_lib.TTT_ERR_INVALID_ARG, "ttt_softce_workspace_size")
    return int(n)


def softce_fwd(h, W, y, *, cu_seqlens=None, loss_mask=None, pass_weight=None, pass_count=None,
               workspace: Optional[torch.Tensor] = None, events=None, out=None, row_teacher=None, row_group=None,
               ngroups: int = 1):
    """Forward: returns (loss [G + 1] = per-pass (per-group) losses then their sum,
    row_loss [P, T], lse [2, P, T] = logsumexp of each row's logits and of its teacher
    row).  ``out`` = (loss, row_loss, lse) writes into given float32 tensors."""
    desc = make_desc(h, W, y, cu_seqlens, loss_mask, pass_weight, pass_count, 0, events, row_teacher, row_group,
                     ngroups)
    P, T, G = desc.P, desc.T, ngroups_of(desc)
    dev = h.device
    if out is None:
        loss = torch.empty(G + 1, dtype=torch.float32, device=dev)
        row_loss = torch.empty(P, T, dtype=torch.float32, device=dev)
        lse = torch.empty(2, P, T, dtype=torch.float32, device=dev)
    else:
        loss, row_loss, lse = out
        for t, shape in ((loss, (G + 1,)), (row_loss, (P, T)), (lse, (2, P, T))):
            if t.dtype != torch.float32 or tuple(t.shape) != shape or not t.is_contiguous():
                raise ValueError(f"out tensors must be contiguous float32 of shapes {(G + 1,)}, {(P, T)}, {(2, P, T)}")
    need = workspace_bytes(desc, False)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _lib.check(_lib.lib().ttt_softce_fwd(ctypes.byref(desc), _ptr(h), _ptr(W), _ptr(y), _ptr(row_loss), _ptr(lse),
                                         _ptr(loss), _ptr(workspace), workspace.numel(), _stream()),
               "ttt_softce_fwd")
    return loss, row_loss, lse


def softce_bwd(h, W, y, lse, *, grad: float = 1.0, cu_seqlens=None, loss_mask=None, pass_weight=None,
               pass_count=None, token_chunk_size: int = 0, with_dw: bool = True, dW=None, dh=None,
               workspace: Optional[torch.Tensor] = None, events=None, row_teacher=None, row_group=None,
               ngroups: int = 1):
    """Backward of grad * L: returns (dh [P, T, d] bf16, dW [V, d] fp32 or None).  A given
    ``dW`` (fp32 [V, d]) is added to; otherwise a zeroed one is allocated.  A given ``dh``
    (bf16 like h) is written."""
    desc = make_desc(h, W, y, cu_seqlens, loss_mask, pass_weight, pass_count, token_chunk_size, events,
                     row_teacher, row_group, ngroups)
    if lse.dtype != torch.float32 or tuple(lse.shape) != (2, desc.P, desc.T) or not lse.is_contiguous():
        raise ValueError("lse must be the forward's float32 [2, P, T]")
    dev = h.device
    if dh is None:
        dh = torch.empty_like(h)
    elif dh.dtype != torch.bfloat16 or dh.shape != h.shape or not dh.is_contiguous():
        raise ValueError("dh must be a contiguous bf16 tensor shaped like h")
    if with_dw and dW is None:
        dW = torch.zeros(desc.V, desc.d, dtype=torch.float32, device=dev)
    if dW is not None and (dW.dtype != torch.float32 or tuple(dW.shape) != (desc.V, desc.d)
                           or not dW.is_contiguous()):
        raise ValueError("dW must be a contiguous float32 [V, d]")
    need = workspace_bytes(desc, True)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _lib.check(_lib.lib().ttt_softce_bwd(ctypes.byref(desc), _ptr(h), _ptr(W), _ptr(y), _ptr(lse),
                                         ctypes.c_float(grad), _ptr(dh), _ptr(dW), _ptr(workspace),
                                         workspace.numel(), _stream()),
               "ttt_softce_bwd")
    return dh, dW


def softce_fwd_bwd(h, W, y, *, grad: float = 1.0, cu_seqlens=None, loss_mask=None, pass_weight=None,
                   pass_count=None, token_chunk_size: int = 0, with_dw: bool = True, dW=None, dh=None, out=None,
                   workspace: Optional[torch.Tensor] = None, events=None, row_teacher=None, row_group=None,
                   ngroups: int = 1):
    """Forward and backward of grad * L in one sweep (the logits GEMM runs once): returns
    (loss, row_loss, lse, dh, dW), the outputs of :func:`softce_fwd` and :func:`softce_bwd`."""
    desc = make_desc(h, W, y, cu_seqlens, loss_mask, pass_weight, pass_count, token_chunk_size, events,
                     row_teacher, row_group, ngroups)
    P, T, G = desc.P, desc.T, ngroups_of(desc)
    dev = h.device
    if out is None:
        loss = torch.empty(G + 1, dtype=torch.float32, device=dev)
        row_loss = torch.empty(P, T, dtype=torch.float32, device=dev)
        lse = torch.empty(2, P, T, dtype=torch.float32, device=dev)
    else:
        loss, row_loss, lse = out
        for t, shape in ((loss, (G + 1,)), (row_loss, (P, T)), (lse, (2, P, T))):
            if t.dtype != torch.float32 or tuple(t.shape) != shape or not t.is_contiguous():
                raise ValueError(f"out tensors must be contiguous float32 of shapes {(G + 1,)}, {(P, T)}, {(2, P, T)}")
    if dh is None:
        dh = torch.empty_like(h)
    elif dh.dtype != torch.bfloat16 or dh.shape != h.shape or not dh.is_contiguous():
        raise ValueError("dh must be a contiguous bf16 tensor shaped like h")
    if with_dw and dW is None:
        dW = torch.zeros(desc.V, desc.d, dtype=torch.float32, device=dev)
    if dW is not None and (dW.dtype != torch.float32 or tuple(dW.shape) != (desc.V, desc.d)
                           or not dW.is_contiguous()):
        raise ValueError("dW must be a contiguous float32 [V, d]")
    need = workspace_bytes(desc, 2)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _lib.check(_lib.lib().ttt_softce_fwd_bwd(ctypes.byref(desc), _ptr(h), _ptr(W), _ptr(y), ctypes.c_float(grad),
                                             _ptr(row_loss), _ptr(lse), _ptr(loss), _ptr(dh), _ptr(dW),
                                             _ptr(workspace), workspace.numel(), _stream()),
               "ttt_softce_fwd_bwd")
    return loss, row_loss, lse, dh, dW


def device_status(workspace: torch.Tensor) -> tuple:
    """(status, detail) of the bounded in-kernel waits of the calls made with ``workspace``."""
    detail = ctypes.c_uint32(0)
    st = _lib.lib().ttt_attn_device_status(_ptr(workspace), _stream(), ctypes.byref(detail))
    return int(st), int(detail.value)
