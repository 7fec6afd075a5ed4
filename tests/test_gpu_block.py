"""GPU parity of the block-draft attention (DFlash/DSpark anchor + mask-token blocks):
the CUDA path through the C ABI against the fp64 block-draft oracle on the same seeded
inputs.  Tolerances as for the TTT attention: O max-abs <= 2e-2, lse max-abs <= 1e-3,
gradient relative L2 <= 1e-2 (each of dqb, dk_ctx, dv_ctx, dkb, dvb on its own)."""

import numpy as np
import pytest
import torch

import ttt_inputs
from tests import block_parity as bp

pytestmark = pytest.mark.gpu

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def _check(w, scale=None, window=0, **kw):
    inp = ttt_inputs.make_block_inputs(w)
    gpu = bp.run_gpu(w, inp, scale=scale, window=window)
    m = bp.compare(w, inp, gpu, scale=scale, window=window, **kw)
    print(w.name, m)
    bp.assert_within(m)
    return m


@needs_cuda
def test_block_tiny_full():
    """B=1, context 128, 8 blocks of 4 tokens, 4/2 heads, D=64: every element."""
    _check(ttt_inputs.block_workloads()["block_tiny"])


@needs_cuda
@pytest.mark.parametrize("Bs,D", [(1, 128), (16, 128), (7, 64), (16, 64)])
def test_block_ragged_thd(Bs, D):
    """Packed batch: contexts of 1, 130, 300, 64 and 257 tokens with 1, 9, 17, 0 and 5
    blocks; anchors at the first and the last context position included (the 1-token
    context can only anchor at 0); block sizes 1 (a plain truncated-causal row), 7 and 16
    (the largest)."""
    ctx = [1, 130, 300, 64, 257]
    nblk = [1, 9, 17, 0, 5]
    import random
    rng = random.Random(Bs * 100 + D)
    anchors = []
    for L, nb in zip(ctx, nblk):
        a = sorted([0, L - 1] + [rng.randrange(L) for _ in range(max(nb - 2, 0))])[:nb] if nb else []
        if nb == 1:
            a = [L - 1]
        anchors += a
    w = ttt_inputs.block_thd(f"block_ragged_bs{Bs}", ctx, nblk, Bs, 8, 2, D, 1e4, anchors=anchors)
    _check(w)


@needs_cuda
def test_block_dense_anchor_edges():
    """Dense: anchors at 0, at tile edges (127, 128) and at the last position, repeated
    anchors (blocks with the same truncation), 3 sequences."""
    anchors = [0, 0, 127, 128, 255, 299] * 3
    w = ttt_inputs.block_dense("block_edges", 3, 300, 6, 5, 4, 4, 128, 1e6, anchors=anchors)
    _check(w)


@needs_cuda
def test_block_non_default_scale():
    w = ttt_inputs.block_thd("block_scale", [200, 90], [6, 3], 8, 4, 2, 128, 1e4)
    _check(w, scale=0.37 / 128 ** 0.5)


@needs_cuda
def test_block_4k_sampled_group():
    """B=2, context 4096, 256 blocks of 16 per sequence, 32/8 heads, D=128, theta 1e6: the
    full tensors of sequence 1 and KV head 6 (its 4 query heads) against the oracle."""
    _check(ttt_inputs.block_workloads()["block_draft_4k"], kv_heads=[6], seqs=[1])


@needs_cuda
def test_block_reuse_rotation_and_deterministic():
    """One workspace for both calls with the backward reusing the forward's rotation, and
    the ordered dq: gradients bit-identical across two backward runs and within the
    tolerances."""
    w = ttt_inputs.block_thd("block_det", [300, 129], [17, 6], 16, 8, 2, 128, 1e4)
    inp = ttt_inputs.make_block_inputs(w)
    a = bp.run_gpu(w, inp, reuse_rotation=True, deterministic=True)
    b = bp.run_gpu(w, inp, reuse_rotation=True, deterministic=True)
    for n in ("dqb", "dk_ctx", "dv_ctx", "dkb", "dvb"):
        assert torch.equal(a[n], b[n]), n
    m = bp.compare(w, inp, a)
    print("reuse+deterministic", m)
    bp.assert_within(m)


@needs_cuda
def test_block_autograd():
    from attention_pass_rope_b200 import ops
    w = ttt_inputs.block_thd("block_autograd", [70, 200], [3, 4], 4, 4, 2, 64, 1e4)
    inp = ttt_inputs.make_block_inputs(w)
    t, kw = bp.gpu_tensors(w, inp)
    leaves = {n: t[n].clone().requires_grad_(True) for n in ("k_ctx", "v_ctx", "qb", "kb", "vb")}
    o = ops.block_attention(leaves["k_ctx"], leaves["v_ctx"], leaves["qb"], leaves["kb"], leaves["vb"],
                            t["anchors"], theta=w.theta, **kw)
    o.backward(t["do"])
    _, lse = ops.block_attn_fwd(*(t[n] for n in ("k_ctx", "v_ctx", "qb", "kb", "vb", "anchors")), theta=w.theta,
                                **kw)
    torch.cuda.synchronize()
    gpu = {"o": o.detach(), "lse": lse, "dk_ctx": leaves["k_ctx"].grad, "dv_ctx": leaves["v_ctx"].grad,
           "dqb": leaves["qb"].grad, "dkb": leaves["kb"].grad, "dvb": leaves["vb"].grad}
    m = bp.compare(w, inp, gpu)
    bp.assert_within(m)


@needs_cuda
def test_block_unsorted_anchors_reported():
    """The backward walks the query tiles in anchor order: anchors that decrease within a
    sequence are an argument error, reported by the status call; the forward stays
    exact for any order."""
    from attention_pass_rope_b200 import ops, _lib
    anchors = [50, 10, 120, 3]
    w = ttt_inputs.block_thd("block_unsorted", [130], [4], 4, 4, 2, 128, 1e4, anchors=anchors)
    inp = ttt_inputs.make_block_inputs(w)
    gpu = bp.run_gpu(w, inp, with_grad=False)
    m = bp.compare(w, inp, gpu, with_grad=False)
    bp.assert_within(m)
    t, kw = bp.gpu_tensors(w, inp)
    args = [t[n] for n in ("k_ctx", "v_ctx", "qb", "kb", "vb", "anchors")]
    lay = ops._block_layout(*args, kw["cu_ctx"], kw["cu_blocks"], kw["max_ctx"], kw["max_blocks"])
    ws = ops.alloc_workspace(ops.block_workspace_bytes(lay, t["anchors"], w.theta, for_backward=True), "cuda")
    o, lse = ops.block_attn_fwd(*args, theta=w.theta, workspace=ws, **kw)
    ops.block_attn_bwd(*args, o, lse, t["do"], theta=w.theta, workspace=ws, **kw)
    st, word = ops.device_status(ws)
    assert st == _lib.TTT_ERR_INVALID_ARG and word == 0x72000001


# ----------------------------------------------------------------------------- sliding-window layers
def _ragged_anchors(ctx, nblk, seed):
    import random
    rng = random.Random(seed)
    anchors = []
    for L, nb in zip(ctx, nblk):
        a = sorted([0, L - 1] + [rng.randrange(L) for _ in range(max(nb - 2, 0))])[:nb] if nb else []
        if nb == 1:
            a = [L - 1]
        anchors += a
    return anchors


@needs_cuda
@pytest.mark.parametrize("window", [1, 50, 129, 1000])
def test_block_window_ragged_thd(window):
    """Sliding-window layers on the packed batch of test_block_ragged_thd (Bs = 16,
    D = 128): a window of 1 (the anchor's key alone), 50 and 129 (trunk ranges that start
    inside a key tile and cross tile edges), and 1000 (longer than every context: the
    full layer)."""
    ctx = [1, 130, 300, 64, 257]
    nblk = [1, 9, 17, 0, 5]
    w = ttt_inputs.block_thd(f"block_window{window}", ctx, nblk, 16, 8, 2, 128, 1e4,
                             anchors=_ragged_anchors(ctx, nblk, 7))
    _check(w, window=window)


@needs_cuda
@pytest.mark.parametrize("window", [128, 200])
def test_block_window_dense_edges(window):
    """Dense, anchors at 0, at the tile edges 127 / 128 and at the last position, with
    windows of exactly one key tile and of a tile and a half (D = 64, Bs = 5)."""
    anchors = [0, 0, 127, 128, 255, 299] * 3
    w = ttt_inputs.block_dense(f"block_window_edges{window}", 3, 300, 6, 5, 4, 4, 64, 1e6, anchors=anchors)
    _check(w, window=window)


@needs_cuda
def test_block_window_4k_sampled_group():
    """The 4K block workload as a sliding-window layer of 1024 keys: sequence 0, KV head
    3 against the oracle."""
    _check(ttt_inputs.block_workloads()["block_draft_4k"], window=1024, kv_heads=[3], seqs=[0])


def _random_block_config(seed):
    """A seeded random packed block-draft configuration: 1-4 sequences with contexts of
    1-300 tokens and 0-12 blocks each at sorted random anchors (repeats allowed), Bs in
    1..16, D in {64, 128}, 1-2 KV heads with groups of 1-4, and a sliding window (0 = the
    full layer) half of the time."""
    rng = np.random.default_rng(seed)
    nseq = int(rng.integers(1, 5))
    ctx = [int(x) for x in rng.integers(1, 301, nseq)]
    nblk = [int(x) for x in rng.integers(0, 13, nseq)]
    if sum(nblk) == 0:
        nblk[0] = 1
    anchors = []
    for L, nb in zip(ctx, nblk):
        anchors += sorted(int(a) for a in rng.integers(0, L, nb))
    Hkv = int(rng.integers(1, 3))
    H = Hkv * int(rng.integers(1, 5))
    window = int(rng.integers(1, 200)) if rng.random() < 0.5 else 0
    return dict(ctx=ctx, nblk=nblk, anchors=anchors, Bs=int(rng.integers(1, 17)), H=H, Hkv=Hkv,
                D=int(rng.choice([64, 128])), window=window)


@needs_cuda
@pytest.mark.parametrize("seed", range(6))
def test_block_random_configurations(seed):
    """Seeded random combinations of the block-draft parameters, every element against the
    oracle."""
    c = _random_block_config(2000 + seed)
    w = ttt_inputs.block_thd(f"block_random{seed}", c["ctx"], c["nblk"], c["Bs"], c["H"], c["Hkv"], c["D"], 1e4,
                             anchors=c["anchors"])
    _check(w, window=c["window"])
