"""ttt_attn_fwd_noalloc: the forward for callers that cannot allocate device memory
(for example a plugin whose host framework owns every device allocation, or a
latency-critical loop where cudaMalloc would synchronise the device).  It keeps its
scratch in a fixed 32 MiB array inside the library instead of a caller workspace.

It runs the same kernels as ttt_attn_fwd on the same inputs, so its outputs must be
bit-identical to that entry point's, on consecutive calls that share the array (a
stale value left in the array by the previous call would show up as a difference).
Its bounded-wait status word lives in the array too and is read with
ttt_attn_fwd_noalloc_status.  This file is collected last on purpose."""

import ctypes

import pytest
import torch

import ttt_inputs
from attention_pass_rope_b200 import _lib, build, ops
from tests import parity


def _lib_built():
    build.build()
    return _lib.lib()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """A workspace need above 32 MiB is refused before anything is enqueued."""
    L = _lib_built()
    w = ttt_inputs.workloads()["qwen3_8b_4k"]
    lay = ops.Layout(w.P, w.H, w.Hkv, w.D, True, B=2, S=4096, T=8192, nseq=2, max_seqlen=4096)
    d = ops.make_desc(lay, w.theta, None)
    fake = ctypes.c_void_p(1 << 20)
    assert L.ttt_attn_fwd_noalloc(ctypes.byref(d), fake, fake, fake, fake, fake, None) == _lib.TTT_ERR_WORKSPACE
    lay.D = 96
    d = ops.make_desc(lay, w.theta, None)
    assert L.ttt_attn_fwd_noalloc(ctypes.byref(d), fake, fake, fake, fake, fake, None) == _lib.TTT_ERR_UNSUPPORTED


needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


@pytest.mark.gpu
@needs_cuda
@pytest.mark.parametrize("w", [ttt_inputs.workloads()["tiny"],
                               ttt_inputs.thd("ragged", [1, 70, 129, 257], 3, 4, 2, 128, 1e4)],
                         ids=["tiny", "thd_ragged"])
def test_noalloc_matches_workspace_forward_twice(w):
    L = _lib_built()
    inp = ttt_inputs.make_inputs(w, with_grad=False)
    q, k, v, _, cu = parity.gpu_shapes(w, inp)
    kw = dict(theta=w.theta, cu_seqlens=cu, max_seqlen=None if w.dense else w.max_seqlen)
    o_ref, lse_ref = ops.ttt_attn_fwd(q, k, v, **kw)
    lay = ops._layout(q, k, v, cu, kw["max_seqlen"])
    desc = ops.make_desc(lay, w.theta, None)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        o = torch.full_like(q, float("nan"))
        lse = torch.full(lay.lse_shape, float("nan"), dtype=torch.float32, device=q.device)
        st = L.ttt_attn_fwd_noalloc(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                    lse.data_ptr(), stream)
        assert st == _lib.TTT_OK, _lib.status_string(st)
        word = ctypes.c_uint32(7)
        assert L.ttt_attn_fwd_noalloc_status(stream, ctypes.byref(word)) == _lib.TTT_OK and word.value == 0
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


@pytest.mark.gpu
@needs_cuda
def test_noalloc_status_reports_a_timed_out_wait():
    """A bounded wait whose status word is the scratch array's gives up and is reported by
    ttt_attn_fwd_noalloc_status as TTT_ERR_DEVICE_TIMEOUT, once (the word is cleared)."""
    L = _lib_built()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.ttt_attn_noalloc_watchdog_selftest(2_000_000, stream) == _lib.TTT_OK
    word = ctypes.c_uint32(0)
    assert L.ttt_attn_fwd_noalloc_status(stream, ctypes.byref(word)) == _lib.TTT_ERR_DEVICE_TIMEOUT
    assert word.value == 0x71000001
    assert L.ttt_attn_fwd_noalloc_status(stream, ctypes.byref(word)) == _lib.TTT_OK and word.value == 0
