"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the same
seeded inputs.  Tolerances: O max-abs <= 2e-2, lse max-abs <= 1e-3, dq/dk/dv
relative L2 <= 1e-2 (bf16 inputs, fp32 accumulation)."""

import numpy as np
import pytest
import torch

import ttt_inputs
from oracle import ttt_oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def _check(w, kv_heads=None, seqs=None, with_grad=True):
    inp = ttt_inputs.make_inputs(w)
    gpu = parity.run_gpu(w, inp, with_grad=with_grad)
    m = parity.compare_full(w, inp, gpu, with_grad=with_grad, kv_heads=kv_heads, seqs=seqs)
    print(w.name, m)
    parity.assert_within(m)
    return m


@needs_cuda
def test_tiny_config_full():
    """B=1, S=128, P=3, 4/2 heads, D=64, theta 1e4: every output element."""
    _check(ttt_inputs.workloads()["tiny"])


@needs_cuda
@pytest.mark.parametrize("P,H,Hkv,D,lengths", [
    (3, 4, 2, 64, [1, 5, 130, 257, 64]),
    (1, 2, 2, 128, [200, 3, 129]),
    (4, 8, 2, 128, [300, 128, 17, 1]),
    (2, 3, 1, 128, [70, 260]),
])
def test_packed_ragged(P, H, Hkv, D, lengths):
    """THD with lengths that are not multiples of the tiles (1, 3, 17, 129, 257, ...)."""
    _check(ttt_inputs.thd("ragged", lengths, P, H, Hkv, D, 1e4))


@needs_cuda
@pytest.mark.parametrize("B,S,P,H,Hkv,D", [(2, 200, 3, 4, 4, 128), (3, 64, 5, 2, 1, 64), (1, 384, 2, 8, 2, 128)])
def test_dense_tails(B, S, P, H, Hkv, D):
    _check(ttt_inputs.dense("dense_tail", B, S, P, H, Hkv, D, 1e6))


@needs_cuda
def test_4k_config_sampled_group():
    """B=2, S=4096, P=3, 32/8 heads, D=128, theta 1e6: full tensors of KV head 5
    (its 4 query heads, all passes, both sequences) against the oracle."""
    _check(ttt_inputs.workloads()["qwen3_8b_4k"], kv_heads=[5])


@needs_cuda
def test_rotated_inputs_tiny():
    """Workspace contents after the forward: the rotated q~ / k~ (bf16), head-major,
    against the oracle's fp64 rotation rounded to bf16."""
    from attention_pass_rope_b200 import ops
    w = ttt_inputs.workloads()["tiny"]
    inp = ttt_inputs.make_inputs(w, with_grad=False)
    q, k, v, _, cu = parity.gpu_shapes(w, inp)
    lay = ops._layout(q, k, v, None, None)
    ws = ops.alloc_workspace(ops.workspace_bytes(lay, w.theta), q.device)
    ops.ttt_attn_fwd(q, k, v, theta=w.theta, workspace=ws)
    torch.cuda.synchronize()
    offs = ops.workspace_layout(lay, w.theta)
    assert len(offs) == 3
    P, T, H, Hkv, D = w.P, w.T, w.H, w.Hkv, w.D

    def view(i, n, dtype):
        return ws[offs[i]:offs[i] + n * torch.tensor([], dtype=dtype).element_size()].view(dtype)

    qr = view(1, P * H * T * D, torch.bfloat16).view(P, H, T, D).permute(0, 2, 1, 3)
    kr = view(2, P * Hkv * T * D, torch.bfloat16).view(P, Hkv, T, D).permute(0, 2, 1, 3)
    qn, kn, vn, _ = parity.oracle_np(inp)
    qr_ref, kr_ref = orc.rotate_inputs(qn, kn, w.theta, rope_round="bf16")
    # fp32 rotation vs fp64 rotation, both rounded to bf16: a rare one-ulp flip
    dq_ = np.abs(parity.to64(qr) - qr_ref)
    assert np.mean(dq_ > 0) < 2e-3 and np.max(dq_) <= 2.0 ** -7 * np.max(np.abs(qr_ref))
    dk_ = np.abs(parity.to64(kr) - kr_ref)
    assert np.mean(dk_ > 0) < 2e-3


@needs_cuda
def test_watchdog_timeout_reported():
    """A bounded wait on a barrier that nothing completes gives up after the budget
    and is reported as TTT_ERR_DEVICE_TIMEOUT; the context stays usable."""
    from attention_pass_rope_b200 import ops, _lib
    ws = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    ops.watchdog_selftest(ws, budget_ns=2_000_000)
    st, word = ops.device_status(ws)
    assert st == _lib.TTT_ERR_DEVICE_TIMEOUT
    assert word == 0x71000001
    st, word = ops.device_status(ws)
    assert st == _lib.TTT_OK and word == 0
    # the device still works
    x = torch.ones(16, device="cuda")
    assert float(x.sum()) == 16.0


@needs_cuda
def test_no_device_timeouts_after_calls():
    from attention_pass_rope_b200 import ops, _lib
    w = ttt_inputs.workloads()["tiny"]
    inp = ttt_inputs.make_inputs(w)
    q, k, v, do, _ = parity.gpu_shapes(w, inp)
    lay = ops._layout(q, k, v, None, None)
    ws = ops.alloc_workspace(ops.workspace_bytes(lay, w.theta, for_backward=True), q.device)
    o, lse = ops.ttt_attn_fwd(q, k, v, theta=w.theta, workspace=ws)
    assert ops.device_status(ws)[0] == _lib.TTT_OK
    ops.ttt_attn_bwd(q, k, v, o, lse, do, theta=w.theta, workspace=ws)
    assert ops.device_status(ws)[0] == _lib.TTT_OK
