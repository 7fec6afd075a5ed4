"""ctypes view of libttt_attn.so (declarations in include/ttt_attn.h)."""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libttt_attn.so")

TTT_OK = 0
TTT_ERR_INVALID_ARG = 1
TTT_ERR_UNSUPPORTED = 2
TTT_ERR_WORKSPACE = 3
TTT_ERR_CUDA = 4
TTT_ERR_DEVICE_TIMEOUT = 5

TTT_LAYOUT_BSHD = 0
TTT_LAYOUT_THD = 1

TTT_FLAG_ROTATED_IN_WORKSPACE = 1
TTT_FLAG_DETERMINISTIC_DQ = 2

KERNELS = ("rope_fwd", "trunk_fwd", "unused_2", "rope_bwd", "bwd_preprocess", "trunk_bwd", "branch_bwd")
KERNEL_COUNT = 8


class TTTEvents(ctypes.Structure):
    _fields_ = [("start", ctypes.c_void_p * KERNEL_COUNT), ("stop", ctypes.c_void_p * KERNEL_COUNT)]


class TTTDesc(ctypes.Structure):
    _fields_ = [
        ("layout", ctypes.c_int),
        ("P", ctypes.c_int),
        ("B", ctypes.c_int),
        ("S", ctypes.c_int),
        ("H", ctypes.c_int),
        ("Hkv", ctypes.c_int),
        ("D", ctypes.c_int),
        ("rope_theta", ctypes.c_float),
        ("softmax_scale", ctypes.c_float),
        ("cu_seqlens", ctypes.c_void_p),
        ("nseq", ctypes.c_int),
        ("total_tokens", ctypes.c_int),
        ("max_seqlen", ctypes.c_int),
        ("events", ctypes.c_void_p),
        ("flags", ctypes.c_int),
        ("pass_stride_q", ctypes.c_int64),
        ("pass_stride_kv", ctypes.c_int64),
    ]


class TTTBlockDesc(ctypes.Structure):
    _fields_ = [
        ("layout", ctypes.c_int),
        ("B", ctypes.c_int),
        ("S", ctypes.c_int),
        ("nblk", ctypes.c_int),
        ("H", ctypes.c_int),
        ("Hkv", ctypes.c_int),
        ("D", ctypes.c_int),
        ("Bs", ctypes.c_int),
        ("rope_theta", ctypes.c_float),
        ("softmax_scale", ctypes.c_float),
        ("anchors", ctypes.c_void_p),
        ("cu_ctx", ctypes.c_void_p),
        ("cu_blocks", ctypes.c_void_p),
        ("nseq", ctypes.c_int),
        ("total_ctx", ctypes.c_int),
        ("total_blocks", ctypes.c_int),
        ("max_ctx", ctypes.c_int),
        ("max_blocks", ctypes.c_int),
        ("events", ctypes.c_void_p),
        ("flags", ctypes.c_int),
        ("window", ctypes.c_int),
    ]


class TTTRingDesc(ctypes.Structure):
    _fields_ = [
        ("P", ctypes.c_int),
        ("H", ctypes.c_int),
        ("Hkv", ctypes.c_int),
        ("D", ctypes.c_int),
        ("rope_theta", ctypes.c_float),
        ("softmax_scale", ctypes.c_float),
        ("q_len", ctypes.c_int),
        ("q_start", ctypes.c_int),
        ("kv_len", ctypes.c_int),
        ("kv_start", ctypes.c_int),
        ("include_branch", ctypes.c_int),
    ]


class TTTSoftceDesc(ctypes.Structure):
    _fields_ = [
        ("P", ctypes.c_int),
        ("T", ctypes.c_int),
        ("d", ctypes.c_int),
        ("V", ctypes.c_int),
        ("cu_seqlens", ctypes.c_void_p),
        ("nseq", ctypes.c_int),
        ("loss_mask", ctypes.c_void_p),
        ("pass_weight", ctypes.c_void_p),
        ("pass_count", ctypes.c_void_p),
        ("token_chunk_size", ctypes.c_int),
        ("events", ctypes.c_void_p),
        ("row_teacher", ctypes.c_void_p),
        ("row_group", ctypes.c_void_p),
        ("ngroups", ctypes.c_int),
        ("teacher_rows", ctypes.c_int),
    ]


class TTTError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = f"{what}: {status_string(status)} (status {status})"
        if status == TTT_ERR_CUDA:
            try:
                code = lib().ttt_attn_last_cuda_error()
                msg += f"; CUDA: {lib().ttt_attn_cuda_error_name(code).decode()} ({code})"
            except Exception:  # pragma: no cover - only used for messages
                pass
        super().__init__(msg)


_lib = None


def lib() -> ctypes.CDLL:
    """Load the library; raises if it has not been built (there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m attention_pass_rope_b200.build` "
            "(the TTT attention has no other implementation)")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER
    vp, sz, u32, u64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint32, ctypes.c_uint64
    D = P(TTTDesc)
    L.ttt_attn_workspace_size.argtypes = [D, ctypes.c_int]
    L.ttt_attn_workspace_size.restype = sz
    L.ttt_attn_workspace_layout.argtypes = [D, ctypes.c_int, P(sz)]
    L.ttt_attn_workspace_layout.restype = ctypes.c_int
    L.ttt_attn_fwd.argtypes = [D, vp, vp, vp, vp, vp, vp, sz, vp]
    L.ttt_attn_fwd.restype = ctypes.c_int
    L.ttt_attn_bwd.argtypes = [D, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.ttt_attn_bwd.restype = ctypes.c_int
    L.ttt_attn_device_status.argtypes = [vp, vp, P(u32)]
    L.ttt_attn_device_status.restype = ctypes.c_int
    L.ttt_attn_watchdog_selftest.argtypes = [vp, sz, u64, vp]
    L.ttt_attn_watchdog_selftest.restype = ctypes.c_int
    L.ttt_attn_fwd_noalloc.argtypes = [D, vp, vp, vp, vp, vp, vp]
    L.ttt_attn_fwd_noalloc.restype = ctypes.c_int
    L.ttt_attn_fwd_noalloc_status.argtypes = [vp, P(u32)]
    L.ttt_attn_fwd_noalloc_status.restype = ctypes.c_int
    L.ttt_attn_noalloc_watchdog_selftest.argtypes = [u64, vp]
    L.ttt_attn_noalloc_watchdog_selftest.restype = ctypes.c_int
    L.ttt_attn_set_wait_budget_ns.argtypes = [u64]
    L.ttt_attn_set_wait_budget_ns.restype = None
    BD = P(TTTBlockDesc)
    L.ttt_block_workspace_size.argtypes = [BD, ctypes.c_int]
    L.ttt_block_workspace_size.restype = sz
    L.ttt_block_workspace_layout.argtypes = [BD, ctypes.c_int, P(sz)]
    L.ttt_block_workspace_layout.restype = ctypes.c_int
    L.ttt_block_attn_fwd.argtypes = [BD, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.ttt_block_attn_fwd.restype = ctypes.c_int
    L.ttt_block_attn_bwd.argtypes = [BD] + [vp] * 14 + [sz, vp]
    L.ttt_block_attn_bwd.restype = ctypes.c_int
    RD = P(TTTRingDesc)
    L.ttt_ring_rotate.argtypes = [RD, vp, vp, vp, vp, vp]
    L.ttt_ring_rotate.restype = ctypes.c_int
    L.ttt_ring_step.argtypes = [RD, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.ttt_ring_step.restype = ctypes.c_int
    L.ttt_ring_merge.argtypes = [RD, vp, vp, vp, vp, ctypes.c_int, vp]
    L.ttt_ring_merge.restype = ctypes.c_int
    L.ttt_ring_finish.argtypes = [RD, vp, vp, vp]
    L.ttt_ring_finish.restype = ctypes.c_int
    L.ttt_ring_bwd_workspace_size.argtypes = [RD]
    L.ttt_ring_bwd_workspace_size.restype = ctypes.c_size_t
    L.ttt_ring_bwd_prepare.argtypes = [RD, vp, vp, vp, vp, ctypes.c_size_t, vp]
    L.ttt_ring_bwd_prepare.restype = ctypes.c_int
    L.ttt_ring_bwd_step.argtypes = [RD, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    L.ttt_ring_bwd_step.restype = ctypes.c_int
    L.ttt_ring_bwd_finish.argtypes = [RD, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    L.ttt_ring_bwd_finish.restype = ctypes.c_int
    L.ttt_ring_dkv_finish.argtypes = [RD, vp, vp, vp, vp, vp]
    L.ttt_ring_dkv_finish.restype = ctypes.c_int
    CD = P(TTTSoftceDesc)
    L.ttt_softce_workspace_size.argtypes = [CD, ctypes.c_int]
    L.ttt_softce_workspace_size.restype = sz
    L.ttt_softce_fwd.argtypes = [CD, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.ttt_softce_fwd.restype = ctypes.c_int
    L.ttt_softce_bwd.argtypes = [CD, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp, sz, vp]
    L.ttt_softce_bwd.restype = ctypes.c_int
    L.ttt_softce_fwd_bwd.argtypes = [CD, vp, vp, vp, ctypes.c_float, vp, vp, vp, vp, vp, vp, sz, vp]
    L.ttt_softce_fwd_bwd.restype = ctypes.c_int
    L.ttt_status_string.argtypes = [ctypes.c_int]
    L.ttt_status_string.restype = ctypes.c_char_p
    L.ttt_attn_version.argtypes = []
    L.ttt_attn_version.restype = ctypes.c_char_p
    L.ttt_attn_last_cuda_error.argtypes = []
    L.ttt_attn_last_cuda_error.restype = ctypes.c_int
    L.ttt_attn_cuda_error_name.argtypes = [ctypes.c_int]
    L.ttt_attn_cuda_error_name.restype = ctypes.c_char_p
    _lib = L
    return L


def status_string(status: int) -> str:
    try:
        return lib().ttt_status_string(status).decode()
    except Exception:  # pragma: no cover - only used for messages
        return "unknown"


def check(status: int, what: str) -> None:
    if status != TTT_OK:
        raise TTTError(status, what)
