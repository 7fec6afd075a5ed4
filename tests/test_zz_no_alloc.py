"""ttt_attn_fwd_noalloc: the forward for callers that cannot allocate device memory
(for example a plugin whose host framework owns every device allocation, or a
latency-critical loop where cudaMalloc would synchronise the device).  It keeps its
scratch in a fixed 32 MiB array inside the library instead of a caller workspace.

Its results must equal those of ttt_attn_fwd (same kernels), on consecutive calls
that share the array.  This file is collected last on purpose."""

import ctypes

import numpy as np
import pytest
import torch

import ttt_inputs
from attention_pass_rope_b200 import _lib, build, ops
from tests import parity


def _noalloc():
    build.build()
    f = _lib.lib().ttt_attn_fwd_noalloc
    f.argtypes = [ctypes.POINTER(_lib.TTTDesc)] + [ctypes.c_void_p] * 6
    f.restype = ctypes.c_int
    return f


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """A workspace need above 32 MiB is refused before anything is enqueued."""
    f = _noalloc()
    w = ttt_inputs.workloads()["qwen3_8b_4k"]
    lay = ops.Layout(w.P, w.H, w.Hkv, w.D, True, B=2, S=4096, T=8192, nseq=2, max_seqlen=4096)
    d = ops.make_desc(lay, w.theta, None)
    fake = ctypes.c_void_p(1 << 20)
    assert f(ctypes.byref(d), fake, fake, fake, fake, fake, None) == _lib.TTT_ERR_WORKSPACE
    lay.D = 96
    d = ops.make_desc(lay, w.theta, None)
    assert f(ctypes.byref(d), fake, fake, fake, fake, fake, None) == _lib.TTT_ERR_UNSUPPORTED


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("w", [ttt_inputs.workloads()["tiny"],
                               ttt_inputs.thd("ragged", [1, 70, 129, 257], 3, 4, 2, 128, 1e4)],
                         ids=["tiny", "thd_ragged"])
def test_noalloc_matches_workspace_forward_twice(w):
    f = _noalloc()
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
        st = f(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), stream)
        assert st == _lib.TTT_OK, _lib.status_string(st)
        torch.cuda.synchronize()
        assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
        assert float((o.float() - o_ref.float()).abs().max()) <= parity.O_MAX_ABS
        assert float((lse - lse_ref).abs().max()) <= parity.LSE_MAX_ABS
