"""PyTorch-facing calls of the TTT trunk+branch attention.

Argument marshalling only: tensors are checked for dtype/shape/device/contiguity,
outputs and the workspace are allocated with torch, and the C ABI of
libttt_attn.so is called on the current CUDA stream.  Every arithmetic step runs in
the library's kernels; there is no other implementation to fall back to.

Shapes (pass-major, trunk = index 0 along P):
  dense:  q [P, B, S, H, D], k/v [P, B, S, Hkv, D]    -> o like q, lse [P, B, H, S]
  packed: q [P, T, H, D],    k/v [P, T, Hkv, D] with cu_seqlens (int32, cuda)
                                                      -> o like q, lse [P, H, T]
Each pass of a tensor must be contiguous; the passes themselves may sit at any common
stride (a multiple of 8 elements, no overlap), e.g. slices of one larger buffer that a
caller filled one pass at a time: q, o, dout, dq share one pass stride, k, v, dk, dv
another.  Outputs that are not given are allocated at the inputs' pass strides.
"""

from __future__ import annotations

import ctypes
import dataclasses
from typing import Optional

import torch

from . import _lib


@dataclasses.dataclass
class Layout:
    P: int
    H: int
    Hkv: int
    D: int
    dense: bool
    B: int = 0
    S: int = 0
    T: int = 0
    nseq: int = 0
    max_seqlen: int = 0
    cu_seqlens: Optional[torch.Tensor] = None
    stride_q: int = 0    # elements between passes of q-shaped tensors (packed: T*H*D)
    stride_kv: int = 0   # elements between passes of k-shaped tensors (packed: T*Hkv*D)

    @property
    def lse_shape(self):
        return (self.P, self.B, self.H, self.S) if self.dense else (self.P, self.H, self.T)


def pass_stride(t: torch.Tensor) -> int:
    """Elements between consecutive passes of a pass-major tensor whose every pass is
    contiguous (raises otherwise)."""
    if not t[0].is_contiguous():
        raise ValueError("every pass of a tensor must be contiguous")
    if t.shape[0] == 1:
        return t[0].numel()
    st = t.stride(0)
    if st < t[0].numel() or st % 8 != 0:
        raise ValueError(f"pass stride {st} must be a multiple of 8 elements and at least {t[0].numel()}")
    return st


def _layout(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens, max_seqlen) -> Layout:
    if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
        raise TypeError("q, k, v must be bfloat16")
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("q, k, v must be CUDA tensors")
    if cu_seqlens is None:
        if q.dim() != 5:
            raise ValueError("dense q must be [P, B, S, H, D]")
        P, B, S, H, D = q.shape
        Hkv = k.shape[3]
        if k.shape != (P, B, S, Hkv, D) or v.shape != k.shape:
            raise ValueError("k, v must be [P, B, S, Hkv, D]")
        lay = Layout(P, H, Hkv, D, True, B=B, S=S, T=B * S, nseq=B, max_seqlen=S)
    else:
        if q.dim() != 4:
            raise ValueError("packed q must be [P, T, H, D]")
        P, T, H, D = q.shape
        Hkv = k.shape[2]
        if k.shape != (P, T, Hkv, D) or v.shape != k.shape:
            raise ValueError("k, v must be [P, T, Hkv, D]")
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be a 1-D int32 CUDA tensor")
        if max_seqlen is None:
            raise ValueError("max_seqlen is required with cu_seqlens")
        lay = Layout(P, H, Hkv, D, False, T=T, nseq=cu_seqlens.numel() - 1, max_seqlen=int(max_seqlen),
                     cu_seqlens=cu_seqlens.contiguous())
    if q.numel() == 0 or k.numel() == 0:
        return lay
    lay.stride_q = pass_stride(q)
    lay.stride_kv = pass_stride(k)
    if pass_stride(v) != lay.stride_kv:
        raise ValueError("k and v must share one pass stride")
    return lay


def _check_strides(lay: Layout, q_like=(), kv_like=()):
    """Every q-shaped tensor at the layout's q pass stride, every k-shaped one at its kv
    stride (the descriptor carries one stride per kind)."""
    if lay.T == 0:
        return
    for t in q_like:
        if pass_stride(t) != lay.stride_q:
            raise ValueError("q, o, dout and dq must share one pass stride")
    for t in kv_like:
        if pass_stride(t) != lay.stride_kv:
            raise ValueError("k, v, dk and dv must share one pass stride")


def empty_at_pass_stride(like: torch.Tensor, stride: int, dtype=None) -> torch.Tensor:
    """Uninitialised tensor of like's shape whose passes are ``stride`` elements apart."""
    P = like.shape[0]
    per = like[0].numel()
    if P <= 1 or stride == per:
        return torch.empty(like.shape, dtype=dtype or like.dtype, device=like.device)
    buf = torch.empty((P - 1) * stride + per, dtype=dtype or like.dtype, device=like.device)
    inner = torch.empty(like.shape[1:], dtype=buf.dtype, device="meta").stride()
    return buf.as_strided(like.shape, (stride,) + tuple(inner))


def make_desc(lay: Layout, theta: float, scale: Optional[float], events=None, flags: int = 0) -> _lib.TTTDesc:
    d = _lib.TTTDesc()
    d.layout = _lib.TTT_LAYOUT_BSHD if lay.dense else _lib.TTT_LAYOUT_THD
    d.P, d.H, d.Hkv, d.D = lay.P, lay.H, lay.Hkv, lay.D
    d.B, d.S = lay.B, lay.S
    d.rope_theta = float(theta)
    d.softmax_scale = 0.0 if scale is None else float(scale)
    if not lay.dense:
        d.cu_seqlens = lay.cu_seqlens.data_ptr()
        d.nseq, d.total_tokens, d.max_seqlen = lay.nseq, lay.T, lay.max_seqlen
    d.events = ctypes.addressof(events) if events is not None else None
    d.flags = int(flags)
    packed_q, packed_kv = lay.T * lay.H * lay.D, lay.T * lay.Hkv * lay.D
    d.pass_stride_q = 0 if lay.stride_q in (0, packed_q) else lay.stride_q
    d.pass_stride_kv = 0 if lay.stride_kv in (0, packed_kv) else lay.stride_kv
    return d


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def workspace_bytes(lay: Layout, theta: float, scale=None, for_backward=False) -> int:
    d = make_desc(lay, theta, scale)
    n = _lib.lib().ttt_attn_workspace_size(ctypes.byref(d), int(for_backward))
    if n == 0 and lay.T > 0:
        raise _lib.TTTError(_lib.TTT_ERR_INVALID_ARG, "ttt_attn_workspace_size")
    return int(n)


def workspace_layout(lay: Layout, theta: float, scale=None, for_backward=False) -> list:
    d = make_desc(lay, theta, scale)
    offs = (ctypes.c_size_t * 8)()
    n = _lib.lib().ttt_attn_workspace_layout(ctypes.byref(d), int(for_backward), offs)
    return [int(offs[i]) for i in range(n)]


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def ttt_attn_fwd(q, k, v, *, theta: float, scale: Optional[float] = None, cu_seqlens=None, max_seqlen=None,
                 workspace: Optional[torch.Tensor] = None, out=None, events=None):
    """Forward: returns (o, lse).  ``out=(o, lse)`` writes into given tensors."""
    lay = _layout(q, k, v, cu_seqlens, max_seqlen)
    if out is None:
        o = empty_at_pass_stride(q, lay.stride_q)
        lse = torch.empty(lay.lse_shape, dtype=torch.float32, device=q.device)
    else:
        o, lse = out
    _check_strides(lay, q_like=(o,))
    if not lse.is_contiguous():
        raise ValueError("lse must be contiguous")
    desc = make_desc(lay, theta, scale, events)
    L = _lib.lib()
    need = L.ttt_attn_workspace_size(ctypes.byref(desc), 0)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    st = L.ttt_attn_fwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(workspace),
                        workspace.numel() * workspace.element_size(), _stream())
    _lib.check(st, "ttt_attn_fwd")
    return o, lse


def ttt_attn_bwd(q, k, v, o, lse, dout, *, theta: float, scale: Optional[float] = None, cu_seqlens=None,
                 max_seqlen=None, workspace: Optional[torch.Tensor] = None, out=None, events=None,
                 rotated_in_workspace: bool = False, deterministic: bool = False):
    """Backward: returns (dq, dk, dv) with respect to the pre-RoPE q, k, v.
    ``rotated_in_workspace``: ``workspace`` still holds what ``ttt_attn_fwd`` wrote
    into it for these q, k (TTT_FLAG_ROTATED_IN_WORKSPACE); the rotation is reused.
    ``deterministic``: bitwise reproducible dq (TTT_FLAG_DETERMINISTIC_DQ), slower."""
    if rotated_in_workspace and workspace is None:
        raise ValueError("rotated_in_workspace needs the forward's workspace")
    lay = _layout(q, k, v, cu_seqlens, max_seqlen)
    if dout.dtype != torch.bfloat16 or o.dtype != torch.bfloat16 or lse.dtype != torch.float32:
        raise TypeError("o, dout must be bfloat16 and lse float32")
    if not lse.is_contiguous():
        raise ValueError("lse must be contiguous")
    if out is None:
        dq = empty_at_pass_stride(q, lay.stride_q)
        dk = empty_at_pass_stride(k, lay.stride_kv)
        dv = empty_at_pass_stride(v, lay.stride_kv)
    else:
        dq, dk, dv = out
    _check_strides(lay, q_like=(o, dout, dq), kv_like=(dk, dv))
    flags = (_lib.TTT_FLAG_ROTATED_IN_WORKSPACE if rotated_in_workspace else 0) | \
        (_lib.TTT_FLAG_DETERMINISTIC_DQ if deterministic else 0)
    desc = make_desc(lay, theta, scale, events, flags)
    L = _lib.lib()
    need = L.ttt_attn_workspace_size(ctypes.byref(desc), 1)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    st = L.ttt_attn_bwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq),
                        _ptr(dk), _ptr(dv), _ptr(workspace), workspace.numel() * workspace.element_size(),
                        _stream())
    _lib.check(st, "ttt_attn_bwd")
    return dq, dk, dv


def device_status(workspace: torch.Tensor) -> tuple:
    """(status, raw word) of the bounded in-kernel waits of the last call (synchronises)."""
    word = ctypes.c_uint32(0)
    st = _lib.lib().ttt_attn_device_status(_ptr(workspace), _stream(), ctypes.byref(word))
    return st, word.value


def watchdog_selftest(workspace: torch.Tensor, budget_ns: int) -> int:
    st = _lib.lib().ttt_attn_watchdog_selftest(_ptr(workspace), workspace.numel(), int(budget_ns), _stream())
    _lib.check(st, "ttt_attn_watchdog_selftest")
    return st


def set_wait_budget_ns(budget_ns: int) -> None:
    _lib.lib().ttt_attn_set_wait_budget_ns(int(budget_ns))


class _TTTAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, theta, scale, cu_seqlens, max_seqlen, keep_rotated):
        ws = None
        if keep_rotated:
            lay = _layout(q, k, v, cu_seqlens, max_seqlen)
            ws = alloc_workspace(workspace_bytes(lay, theta, scale, for_backward=True), q.device)
        o, lse = ttt_attn_fwd(q, k, v, theta=theta, scale=scale, cu_seqlens=cu_seqlens, max_seqlen=max_seqlen,
                              workspace=ws)
        ctx.save_for_backward(q, k, v, o, lse, cu_seqlens)
        ctx.theta, ctx.scale, ctx.max_seqlen = theta, scale, max_seqlen
        ctx.has_cu = cu_seqlens is not None
        ctx.ws = ws
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse, cu = ctx.saved_tensors
        if do.shape[0] > 0 and do.numel() > 0:
            try:
                same = pass_stride(do) == pass_stride(o)
            except ValueError:
                same = False
            if not same:
                do = empty_at_pass_stride(o, pass_stride(o)).copy_(do)
        dq, dk, dv = ttt_attn_bwd(q, k, v, o, lse, do, theta=ctx.theta, scale=ctx.scale,
                                  cu_seqlens=cu if ctx.has_cu else None, max_seqlen=ctx.max_seqlen,
                                  workspace=ctx.ws, rotated_in_workspace=ctx.ws is not None)
        ctx.ws = None
        return dq, dk, dv, None, None, None, None, None


def ttt_attention(q, k, v, *, theta: float, scale: Optional[float] = None, cu_seqlens=None, max_seqlen=None,
                  keep_rotated: bool = False):
    """Differentiable TTT trunk+branch attention (autograd over the C ABI).
    ``keep_rotated`` holds the forward's workspace (rotated q~ / k~, sized for the
    backward) until the backward, which then skips rotating q and k again: more
    memory between the two calls, one kernel less in the backward."""
    return _TTTAttention.apply(q, k, v, theta, scale, cu_seqlens, max_seqlen, keep_rotated)


# ----------------------------------------------------------------------------- block-draft attention

@dataclasses.dataclass
class BlockLayout:
    """Shapes of a block-draft call.  dense: k_ctx [B, S, Hkv, D], qb [B, nblk, Bs, H, D],
    kb/vb [B, nblk, Bs, Hkv, D], anchors [B, nblk], lse [B, H, nblk*Bs].  packed:
    k_ctx [Tc, Hkv, D], qb [NB, Bs, H, D], kb/vb [NB, Bs, Hkv, D], anchors [NB], lse
    [H, NB*Bs], with cu_ctx / cu_blocks prefix sums (int32, cuda)."""
    H: int
    Hkv: int
    D: int
    Bs: int
    dense: bool
    B: int = 0
    S: int = 0
    nblk: int = 0
    nseq: int = 0
    Tc: int = 0
    NB: int = 0
    max_ctx: int = 0
    max_blocks: int = 0
    cu_ctx: Optional[torch.Tensor] = None
    cu_blocks: Optional[torch.Tensor] = None

    @property
    def lse_shape(self):
        return (self.B, self.H, self.nblk * self.Bs) if self.dense else (self.H, self.NB * self.Bs)


def _block_layout(k_ctx, v_ctx, qb, kb, vb, anchors, cu_ctx, cu_blocks, max_ctx, max_blocks) -> BlockLayout:
    for t in (k_ctx, v_ctx, qb, kb, vb):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("k_ctx, v_ctx, qb, kb, vb must be contiguous bfloat16 CUDA tensors")
    if anchors.dtype != torch.int32 or not anchors.is_cuda or not anchors.is_contiguous():
        raise ValueError("anchors must be a contiguous int32 CUDA tensor")
    if cu_ctx is None:
        B, S, Hkv, D = k_ctx.shape
        _, nblk, Bs, H, _ = qb.shape
        if qb.shape[:1] != (B,) or qb.shape[4] != D or kb.shape != (B, nblk, Bs, Hkv, D) or vb.shape != kb.shape \
                or v_ctx.shape != k_ctx.shape or anchors.shape != (B, nblk):
            raise ValueError("inconsistent dense block-draft shapes")
        return BlockLayout(H, Hkv, D, Bs, True, B=B, S=S, nblk=nblk, nseq=B, Tc=B * S, NB=B * nblk)
    Tc, Hkv, D = k_ctx.shape
    NB, Bs, H, _ = qb.shape
    if kb.shape != (NB, Bs, Hkv, D) or vb.shape != kb.shape or v_ctx.shape != k_ctx.shape or \
            anchors.shape != (NB,) or qb.shape[3] != D:
        raise ValueError("inconsistent packed block-draft shapes")
    for c in (cu_ctx, cu_blocks):
        if c is None or c.dtype != torch.int32 or not c.is_cuda or c.dim() != 1:
            raise ValueError("cu_ctx and cu_blocks must be 1-D int32 CUDA tensors")
    if max_ctx is None or max_blocks is None:
        raise ValueError("max_ctx and max_blocks are required with cu_ctx / cu_blocks")
    return BlockLayout(H, Hkv, D, Bs, False, nseq=cu_ctx.numel() - 1, Tc=Tc, NB=NB, max_ctx=int(max_ctx),
                       max_blocks=int(max_blocks), cu_ctx=cu_ctx.contiguous(), cu_blocks=cu_blocks.contiguous())


def make_block_desc(lay: BlockLayout, anchors, theta: float, scale: Optional[float], events=None,
                    flags: int = 0, window: int = 0) -> _lib.TTTBlockDesc:
    d = _lib.TTTBlockDesc()
    d.layout = _lib.TTT_LAYOUT_BSHD if lay.dense else _lib.TTT_LAYOUT_THD
    d.B, d.S, d.nblk = lay.B, lay.S, lay.nblk
    d.H, d.Hkv, d.D, d.Bs = lay.H, lay.Hkv, lay.D, lay.Bs
    d.rope_theta = float(theta)
    d.softmax_scale = 0.0 if scale is None else float(scale)
    d.anchors = anchors.data_ptr() if anchors is not None else None
    if not lay.dense:
        d.cu_ctx, d.cu_blocks = lay.cu_ctx.data_ptr(), lay.cu_blocks.data_ptr()
        d.nseq, d.total_ctx, d.total_blocks = lay.nseq, lay.Tc, lay.NB
        d.max_ctx, d.max_blocks = lay.max_ctx, lay.max_blocks
    d.events = ctypes.addressof(events) if events is not None else None
    d.flags = int(flags)
    d.window = int(window or 0)
    return d


def block_workspace_bytes(lay: BlockLayout, anchors, theta: float, scale=None, for_backward=False) -> int:
    d = make_block_desc(lay, anchors, theta, scale)
    n = _lib.lib().ttt_block_workspace_size(ctypes.byref(d), int(for_backward))
    if n == 0 and lay.NB > 0:
        raise _lib.TTTError(_lib.TTT_ERR_INVALID_ARG, "ttt_block_workspace_size")
    return int(n)


def block_attn_fwd(k_ctx, v_ctx, qb, kb, vb, anchors, *, theta: float, scale: Optional[float] = None, cu_ctx=None,
                   cu_blocks=None, max_ctx=None, max_blocks=None, workspace: Optional[torch.Tensor] = None, out=None,
                   events=None, window: int = 0):
    """Block-draft forward: returns (o, lse).  ``window`` > 0: a sliding-window layer,
    each block sees the context keys anchor - window + 1 .. anchor."""
    lay = _block_layout(k_ctx, v_ctx, qb, kb, vb, anchors, cu_ctx, cu_blocks, max_ctx, max_blocks)
    if out is None:
        o = torch.empty_like(qb)
        lse = torch.empty(lay.lse_shape, dtype=torch.float32, device=qb.device)
    else:
        o, lse = out
    desc = make_block_desc(lay, anchors, theta, scale, events, window=window)
    L = _lib.lib()
    if workspace is None:
        workspace = alloc_workspace(L.ttt_block_workspace_size(ctypes.byref(desc), 0), qb.device)
    st = L.ttt_block_attn_fwd(ctypes.byref(desc), _ptr(k_ctx), _ptr(v_ctx), _ptr(qb), _ptr(kb), _ptr(vb), _ptr(o),
                              _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream())
    _lib.check(st, "ttt_block_attn_fwd")
    return o, lse


def block_attn_bwd(k_ctx, v_ctx, qb, kb, vb, anchors, o, lse, dout, *, theta: float, scale: Optional[float] = None,
                   cu_ctx=None, cu_blocks=None, max_ctx=None, max_blocks=None,
                   workspace: Optional[torch.Tensor] = None, out=None, events=None, rotated_in_workspace=False,
                   deterministic=False, window: int = 0):
    """Block-draft backward: returns (dk_ctx, dv_ctx, dqb, dkb, dvb) with respect to the
    pre-RoPE inputs (``window`` as in block_attn_fwd)."""
    if rotated_in_workspace and workspace is None:
        raise ValueError("rotated_in_workspace needs the forward's workspace")
    lay = _block_layout(k_ctx, v_ctx, qb, kb, vb, anchors, cu_ctx, cu_blocks, max_ctx, max_blocks)
    for t in (o, dout):
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.shape != qb.shape:
            raise ValueError("o and dout must be contiguous bfloat16 tensors shaped like qb")
    if lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 tensor")
    if out is None:
        out = tuple(torch.empty_like(t) for t in (k_ctx, v_ctx, qb, kb, vb))
    flags = (_lib.TTT_FLAG_ROTATED_IN_WORKSPACE if rotated_in_workspace else 0) | \
        (_lib.TTT_FLAG_DETERMINISTIC_DQ if deterministic else 0)
    desc = make_block_desc(lay, anchors, theta, scale, events, flags, window)
    L = _lib.lib()
    if workspace is None:
        workspace = alloc_workspace(L.ttt_block_workspace_size(ctypes.byref(desc), 1), qb.device)
    dk_ctx, dv_ctx, dqb, dkb, dvb = out
    st = L.ttt_block_attn_bwd(ctypes.byref(desc), _ptr(k_ctx), _ptr(v_ctx), _ptr(qb), _ptr(kb), _ptr(vb), _ptr(o),
                              _ptr(lse), _ptr(dout), _ptr(dk_ctx), _ptr(dv_ctx), _ptr(dqb), _ptr(dkb), _ptr(dvb),
                              _ptr(workspace), workspace.numel() * workspace.element_size(), _stream())
    _lib.check(st, "ttt_block_attn_bwd")
    return out


class _BlockAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, k_ctx, v_ctx, qb, kb, vb, anchors, theta, scale, cu_ctx, cu_blocks, max_ctx, max_blocks, window):
        o, lse = block_attn_fwd(k_ctx, v_ctx, qb, kb, vb, anchors, theta=theta, scale=scale, cu_ctx=cu_ctx,
                                cu_blocks=cu_blocks, max_ctx=max_ctx, max_blocks=max_blocks, window=window)
        ctx.save_for_backward(k_ctx, v_ctx, qb, kb, vb, anchors, o, lse,
                              *(t for t in (cu_ctx, cu_blocks) if t is not None))
        ctx.kw = dict(theta=theta, scale=scale, max_ctx=max_ctx, max_blocks=max_blocks, window=window)
        ctx.packed = cu_ctx is not None
        return o

    @staticmethod
    def backward(ctx, do):
        saved = ctx.saved_tensors
        k_ctx, v_ctx, qb, kb, vb, anchors, o, lse = saved[:8]
        cu = dict(cu_ctx=saved[8], cu_blocks=saved[9]) if ctx.packed else {}
        grads = block_attn_bwd(k_ctx, v_ctx, qb, kb, vb, anchors, o, lse, do.contiguous(), **cu, **ctx.kw)
        return (*grads, None, None, None, None, None, None, None, None)


def block_attention(k_ctx, v_ctx, qb, kb, vb, anchors, *, theta: float, scale: Optional[float] = None, cu_ctx=None,
                    cu_blocks=None, max_ctx=None, max_blocks=None, window: int = 0):
    """Differentiable block-draft attention (autograd over the C ABI); returns o."""
    return _BlockAttention.apply(k_ctx, v_ctx, qb, kb, vb, anchors, theta, scale, cu_ctx, cu_blocks, max_ctx,
                                 max_blocks, window)
