"""GPU parity of the soft cross-entropy distillation loss (the library's kernels through
the C ABI) against the fp64 oracle, on the same seeded inputs.

Tolerances, from the arithmetic: the logits are fp32 sums of exact bf16 products and the
softmax statistics fp32, so a row's loss and logsumexp are good to ~1e-5 in practice;
LOSS_ATOL allows 1e-3.  The backward rounds dz to bf16 (relative 2^-9 per element)
before the dh and dW GEMMs, so gradients are compared by relative L2 at 1e-2, overall
and per pass."""

import numpy as np
import pytest
import scipy.special
import torch

import ttt_inputs as ti
from attention_pass_rope_b200 import softce as ce
from oracle import softce_oracle as sco

pytestmark = pytest.mark.gpu

LOSS_ATOL = 1e-3
PASS_RTOL = 1e-4
GRAD_RL2 = 1e-2


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _cuda_opt(x, dtype):
    return None if x is None else torch.tensor(x, dtype=dtype, device="cuda")


def run_gpu(inp, cu, *, pass_weight=None, pass_count=None, grad=1.0, chunk=0, mask=True, fused=False):
    h, W, y = inp.h.cuda(), inp.W.cuda(), inp.y.cuda()
    m = inp.mask.cuda() if mask else None
    cu_t = torch.tensor(cu, dtype=torch.int32, device="cuda")
    pw = _cuda_opt(pass_weight, torch.float32)
    pc = _cuda_opt(pass_count, torch.float32)
    kw = dict(cu_seqlens=cu_t, loss_mask=m, pass_weight=pw, pass_count=pc)
    if fused:
        loss, rows, lse, dh, dW = ce.softce_fwd_bwd(h, W, y, grad=grad, token_chunk_size=chunk, **kw)
    else:
        loss, rows, lse = ce.softce_fwd(h, W, y, **kw)
        dh, dW = ce.softce_bwd(h, W, y, lse, grad=grad, token_chunk_size=chunk, **kw)
    torch.cuda.synchronize()
    return loss.cpu().numpy(), rows.cpu().numpy(), lse.cpu().numpy(), dh.float().cpu().numpy(), dW.cpu().numpy()


def compare(inp, cu, out, *, pass_weight=None, pass_count=None, grad=1.0, mask=True):
    loss, rows, lse, dh, dW = out
    P = inp.h.shape[0]
    m = inp.mask.numpy().astype(bool) if mask else None
    ref = sco.forward(inp.h, inp.W, inp.y, cu, m, pass_weight, pass_count)
    idx = sco.teacher_index(cu, P, m)
    valid = idx >= 0
    if valid.any():
        assert np.abs(rows[valid] - ref["rows"][valid]).max() <= LOSS_ATOL
        assert np.abs(lse[0][valid] - ref["lse_z"][valid]).max() <= LOSS_ATOL
        y64 = inp.y.double().numpy()
        lse_y = scipy.special.logsumexp(y64[idx[valid]], axis=1)
        assert np.abs(lse[1][valid] - lse_y).max() <= LOSS_ATOL
    assert np.all(rows[~valid] == 0) and np.all(lse[:, ~valid] == 0)
    np.testing.assert_allclose(loss[:P], ref["pass_loss"], rtol=PASS_RTOL, atol=1e-6)
    assert loss[P] == pytest.approx(ref["loss"], rel=PASS_RTOL, abs=1e-6)
    dh_ref, dW_ref = sco.backward(inp.h, inp.W, inp.y, cu, m, pass_weight, pass_count, grad)
    if np.linalg.norm(dh_ref) == 0:
        assert np.all(dh == 0) and np.all(dW == 0)
        return
    assert rel_l2(dh, dh_ref) <= GRAD_RL2
    for p in range(P):
        if np.linalg.norm(dh_ref[p]) > 0:
            assert rel_l2(dh[p], dh_ref[p]) <= GRAD_RL2, p
        else:
            assert np.all(dh[p] == 0), p
    assert rel_l2(dW, dW_ref) <= GRAD_RL2


def test_softce_tiny():
    w = ti.softce_workloads()["softce_tiny"]
    inp = ti.make_softce_inputs(w)
    compare(inp, w.cu_seqlens, run_gpu(inp, w.cu_seqlens))


def test_softce_tiny_chunks_weights_counts():
    """Ragged backward chunks (100 rows: 7 full chunks and one of 68), pass weights, given
    global counts and an upstream gradient."""
    w = ti.softce_workloads()["softce_tiny"]
    inp = ti.make_softce_inputs(w)
    kw = dict(pass_weight=[1.0, 0.8, 0.64], pass_count=[500.0, 400.0, 300.0], grad=0.5)
    compare(inp, w.cu_seqlens, run_gpu(inp, w.cu_seqlens, chunk=100, **kw), **kw)


def test_softce_mid():
    """Several 128 x 256 tiles in every GEMM, a ragged last vocabulary tile (8200 =
    32 * 256 + 8), eight K slices in the logits GEMM."""
    w = ti.softce_workloads()["softce_mid"]
    inp = ti.make_softce_inputs(w)
    compare(inp, w.cu_seqlens, run_gpu(inp, w.cu_seqlens, chunk=1000))


def test_softce_fused_equals_separate_calls():
    """The fused call gives the separate calls' outputs bit for bit (the same logits, the
    same dz expression, the same GEMMs), and the oracle's values."""
    w = ti.softce_workloads()["softce_tiny"]
    inp = ti.make_softce_inputs(w)
    kw = dict(pass_weight=[1.0, 0.8, 0.64], pass_count=[500.0, 400.0, 300.0], grad=0.5)
    sep = run_gpu(inp, w.cu_seqlens, chunk=100, **kw)
    fus = run_gpu(inp, w.cu_seqlens, chunk=100, fused=True, **kw)
    for a, b in zip(sep, fus):
        assert np.array_equal(a, b)
    compare(inp, w.cu_seqlens, fus, **kw)


def test_softce_fused_mid():
    w = ti.softce_workloads()["softce_mid"]
    inp = ti.make_softce_inputs(w)
    compare(inp, w.cu_seqlens, run_gpu(inp, w.cu_seqlens, chunk=1000, fused=True))


def test_softce_dh_chunk_invariant_and_dw_accumulates():
    w = ti.softce_workloads()["softce_tiny"]
    inp = ti.make_softce_inputs(w)
    h, W, y, m = inp.h.cuda(), inp.W.cuda(), inp.y.cuda(), inp.mask.cuda()
    cu = torch.tensor(w.cu_seqlens, dtype=torch.int32, device="cuda")
    _, _, lse = ce.softce_fwd(h, W, y, cu_seqlens=cu, loss_mask=m)
    dh0, dW0 = ce.softce_bwd(h, W, y, lse, cu_seqlens=cu, loss_mask=m)
    dh1, dW1 = ce.softce_bwd(h, W, y, lse, cu_seqlens=cu, loss_mask=m, token_chunk_size=37)
    torch.cuda.synchronize()
    # a row's dh depends on its own dz row only, reduced in the same order
    assert torch.equal(dh0, dh1)
    assert rel_l2(dW1.cpu().numpy(), dW0.cpu().numpy()) < 1e-5
    # dW is added to
    ce.softce_bwd(h, W, y, lse, cu_seqlens=cu, loss_mask=m, dW=dW1)
    torch.cuda.synchronize()
    assert rel_l2(dW1.cpu().numpy(), 2 * dW0.cpu().numpy()) < 1e-5
    _, none = ce.softce_bwd(h, W, y, lse, cu_seqlens=cu, loss_mask=m, with_dw=False)
    assert none is None


def test_softce_degenerate_cases():
    w = ti.softce_workloads()["softce_tiny"]
    inp = ti.make_softce_inputs(w)
    # every teacher position masked: no valid row, zero losses and gradients
    inp0 = ti.SoftCEInputs(inp.h, inp.W, inp.y, torch.zeros_like(inp.mask))
    out = run_gpu(inp0, w.cu_seqlens)
    assert np.all(out[0] == 0) and np.all(out[1] == 0) and np.all(out[3] == 0) and np.all(out[4] == 0)
    # one-token sequences: only pass 1 has valid rows
    lengths = (1, 1, 1, 1, 1)
    w1 = ti.SoftCEWorkload("one_token", P=3, lengths=lengths, d=64, V=264, seed=3)
    inp1 = ti.make_softce_inputs(w1)
    out1 = run_gpu(inp1, w1.cu_seqlens, mask=False)
    assert out1[0][1] == 0 and out1[0][2] == 0
    compare(inp1, w1.cu_seqlens, out1, mask=False)
    # no tokens at all
    h = torch.zeros(3, 0, 64, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(264, 64, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(0, 264, dtype=torch.bfloat16, device="cuda")
    loss, rows, lse = ce.softce_fwd(h, W, y)
    dh, dW = ce.softce_bwd(h, W, y, lse)
    loss2, _, _, dh2, dW2 = ce.softce_fwd_bwd(h, W, y)
    torch.cuda.synchronize()
    assert loss.abs().sum().item() == 0 and dh.numel() == 0 and dW.abs().sum().item() == 0
    assert loss2.abs().sum().item() == 0 and dW2.abs().sum().item() == 0
    # fused, every position masked
    out0 = run_gpu(inp0, w.cu_seqlens, fused=True)
    assert all(np.all(x == 0) for x in (out0[0], out0[1], out0[3], out0[4]))


def test_softce_ragged_hidden_size():
    """d = 72: a partial last K slice in the logits GEMM (64 + 8), a partial column tile in
    dh and dW, and a partial 32-column slice at the end of the vocabulary (V = 264)."""
    w = ti.SoftCEWorkload("d72", P=2, lengths=(40, 97), d=72, V=264, seed=5)
    inp = ti.make_softce_inputs(w)
    compare(inp, w.cu_seqlens, run_gpu(inp, w.cu_seqlens, chunk=50))
    compare(inp, w.cu_seqlens, run_gpu(inp, w.cu_seqlens, chunk=50, fused=True))


def test_softce_dense_sequences_without_cu_seqlens():
    """A dense batch described by nseq equal sequences (no cu_seqlens): the same results as
    the packed description of the same tokens."""
    import ctypes
    from attention_pass_rope_b200 import _lib
    w = ti.SoftCEWorkload("dense3", P=3, lengths=(60, 60, 60), d=64, V=512, seed=9)
    inp = ti.make_softce_inputs(w)
    h, W, y, m = inp.h.cuda(), inp.W.cuda(), inp.y.cuda(), inp.mask.cuda()
    desc = ce.make_desc(h, W, y, None, m)
    desc.nseq = 3
    P, T = w.P, w.T
    loss = torch.empty(P + 1, device="cuda")
    rows = torch.empty(P, T, device="cuda")
    lse = torch.empty(2, P, T, device="cuda")
    dh = torch.empty_like(h)
    dW = torch.zeros(w.V, w.d, device="cuda")
    ws = torch.empty(ce.workspace_bytes(desc, 2), dtype=torch.uint8, device="cuda")
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    _lib.check(_lib.lib().ttt_softce_fwd_bwd(ctypes.byref(desc), ptr(h), ptr(W), ptr(y), ctypes.c_float(1.0),
                                             ptr(rows), ptr(lse), ptr(loss), ptr(dh), ptr(dW), ptr(ws), ws.numel(),
                                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)),
               "ttt_softce_fwd_bwd")
    torch.cuda.synchronize()
    out = (loss.cpu().numpy(), rows.cpu().numpy(), lse.cpu().numpy(), dh.float().cpu().numpy(), dW.cpu().numpy())
    compare(inp, w.cu_seqlens, out)
    packed = run_gpu(inp, w.cu_seqlens, fused=True)
    for a, b in zip(out, packed):
        assert np.array_equal(a, b)


def test_softce_general_form_equals_pass_form():
    """The TTT passes given as explicit teacher positions and groups: the same rows, lse,
    dh and dW bit for bit as the pass form, and the same per-pass losses (summed in
    another order)."""
    w = ti.softce_workloads()["softce_tiny"]
    inp = ti.make_softce_inputs(w)
    h, W, y, m = inp.h.cuda(), inp.W.cuda(), inp.y.cuda(), inp.mask.cuda()
    cu = torch.tensor(w.cu_seqlens, dtype=torch.int32, device="cuda")
    teacher, group = sco.ttt_mapping(w.cu_seqlens, w.P)
    rt = torch.tensor(teacher, dtype=torch.int32, device="cuda")
    rg = torch.tensor(group, dtype=torch.int32, device="cuda")
    pw = torch.tensor([1.0, 0.7, 0.4], device="cuda")
    a = ce.softce_fwd_bwd(h, W, y, cu_seqlens=cu, loss_mask=m, pass_weight=pw, token_chunk_size=100)
    b = ce.softce_fwd_bwd(h, W, y, loss_mask=m, pass_weight=pw, token_chunk_size=100, row_teacher=rt, row_group=rg,
                          ngroups=w.P)
    c_loss, c_rows, c_lse = ce.softce_fwd(h, W, y, loss_mask=m, pass_weight=pw, row_teacher=rt, row_group=rg,
                                          ngroups=w.P)
    c_dh, c_dW = ce.softce_bwd(h, W, y, c_lse, loss_mask=m, pass_weight=pw, token_chunk_size=100, row_teacher=rt,
                               row_group=rg, ngroups=w.P)
    torch.cuda.synchronize()
    for x, z in zip(a[1:], b[1:]):
        assert torch.equal(x, z)
    assert torch.equal(c_rows, b[1]) and torch.equal(c_lse, b[2]) and torch.equal(c_dh, b[3])
    assert torch.equal(c_dW, b[4])
    assert torch.allclose(a[0], b[0], rtol=1e-6, atol=0) and torch.equal(c_loss, b[0])


def test_softce_block_slots():
    """Block drafters normalised per slot: 40 blocks of 16 slots at sorted anchors over 300
    teacher positions (the last blocks run past them), slot weights, a mask; forward, the
    separate backward and the fused call against the oracle's general form."""
    g = torch.Generator().manual_seed(11)
    nb, Bs, d, V, Ty = 40, 16, 128, 1000, 300
    hq = torch.randn(1, nb * Bs, d, generator=g).to(torch.bfloat16)
    Wq = (torch.randn(V, d, generator=g) * (2.0 / d ** 0.5)).to(torch.bfloat16)
    yq = (torch.randn(Ty, V, generator=g) * 3.0).to(torch.bfloat16)
    mq = (torch.rand(Ty, generator=g) < 0.9).to(torch.uint8)
    anchors = torch.sort(torch.randint(0, Ty, (nb,), generator=g)).values
    teacher = (anchors[:, None] + torch.arange(Bs)[None, :]).reshape(-1).to(torch.int32)
    group = torch.arange(Bs).repeat(nb).to(torch.int32)
    wts = [1.0 / (1 + j) for j in range(Bs)]
    h, W, y, m = hq.cuda(), Wq.cuda(), yq.cuda(), mq.cuda()
    rt, rg = teacher.cuda(), group.cuda()
    pw = torch.tensor(wts, device="cuda")
    kw = dict(loss_mask=m, pass_weight=pw, row_teacher=rt, row_group=rg, ngroups=Bs)
    loss, rows, lse = ce.softce_fwd(h, W, y, **kw)
    dh, dW = ce.softce_bwd(h, W, y, lse, grad=0.8, token_chunk_size=200, **kw)
    f = ce.softce_fwd_bwd(h, W, y, grad=0.8, token_chunk_size=200, **kw)
    torch.cuda.synchronize()
    ref = sco.forward_mapped(hq[0], Wq, yq, teacher.numpy(), group.numpy(), Bs, mq.numpy(), wts)
    dh_ref, dW_ref = sco.backward_mapped(hq[0], Wq, yq, teacher.numpy(), group.numpy(), Bs, mq.numpy(), wts,
                                         grad=0.8)
    valid = ref["valid"]
    assert valid.sum() > 0 and (~valid).sum() > 0
    got_rows = rows.cpu().numpy()[0]
    assert np.abs(got_rows[valid] - ref["rows"][valid]).max() <= LOSS_ATOL
    assert np.all(got_rows[~valid] == 0)
    np.testing.assert_allclose(loss.cpu().numpy()[:Bs], ref["group_loss"], rtol=PASS_RTOL, atol=1e-6)
    assert loss.cpu().numpy()[Bs] == pytest.approx(ref["loss"], rel=PASS_RTOL)
    assert rel_l2(dh.float().cpu().numpy()[0], dh_ref) <= GRAD_RL2
    assert rel_l2(dW.cpu().numpy(), dW_ref) <= GRAD_RL2
    for x, z in zip((loss, rows, lse, dh, dW), f):
        assert torch.equal(x, z)


def _random_softce_config(seed):
    """A seeded random soft-CE configuration: 1-4 sequences of 1-300 tokens, P in 1..4, d a
    multiple of 8 in [64, 320], V a multiple of 8 in [256, 3000], a random chunk size, pass
    weights and upstream gradient, the fused call half of the time."""
    rng = np.random.default_rng(seed)
    nseq = int(rng.integers(1, 5))
    lengths = tuple(int(x) for x in rng.integers(1, 301, nseq))
    P = int(rng.integers(1, 5))
    d = 8 * int(rng.integers(8, 41))
    V = 8 * int(rng.integers(32, 376))
    return dict(w=ti.SoftCEWorkload(f"rnd{seed}", P=P, lengths=lengths, d=d, V=V, seed=seed),
                chunk=int(rng.integers(1, 600)), weights=[float(x) for x in rng.uniform(0.2, 2.0, P)],
                grad=float(rng.uniform(0.5, 2.0)), fused=bool(rng.random() < 0.5))


@pytest.mark.parametrize("seed", range(5))
def test_softce_random_configurations(seed):
    c = _random_softce_config(3000 + seed)
    w = c["w"]
    inp = ti.make_softce_inputs(w)
    kw = dict(pass_weight=c["weights"], grad=c["grad"])
    compare(inp, w.cu_seqlens, run_gpu(inp, w.cu_seqlens, chunk=c["chunk"], fused=c["fused"], **kw), **kw)


@pytest.mark.slow
def test_softce_qwen3_8b_4k_sampled_rows():
    """The full-size workload (P = 3 over 2 x 4096 tokens, d = 4096, V = 151936) in the
    launch configuration that the bench times (the fused call, chunks of 4096 rows): sampled
    rows' losses, logsumexps and dh against the oracle's few-rows forms, and properties
    that hold at any size for the rest."""
    w = ti.softce_workloads()["softce_qwen3_8b_4k"]
    inp = ti.make_softce_inputs(w)
    cu = w.cu_seqlens
    loss, rows, lse, dh, dW = run_gpu(inp, cu, chunk=4096, fused=True)
    P, T = w.P, w.T
    m = inp.mask.numpy().astype(bool)
    idx = sco.teacher_index(cu, P, m)
    counts = (idx >= 0).sum(axis=1)
    # rows at tile edges (127/128 of a 128-row tile), chunk edges (4095/4096) and the ends
    cand = [(0, 0), (0, 127), (0, 128), (1, 4095), (1, 4096), (2, 4094), (2, 8190), (0, 8191), (1, 3000),
            (2, 5000), (0, 6143), (1, 6144)]
    pairs = [(p, t) for p, t in cand if idx[p, t] >= 0]
    assert len(pairs) >= 8
    hr = torch.stack([inp.h[p, t] for p, t in pairs])
    yr = torch.stack([inp.y[idx[p, t]] for p, t in pairs])
    ref_loss, ref_lse = sco.rows_forward(hr, inp.W, yr)
    got_loss = np.array([rows[p, t] for p, t in pairs])
    got_lse = np.array([lse[0, p, t] for p, t in pairs])
    assert np.abs(got_loss - ref_loss).max() <= LOSS_ATOL
    assert np.abs(got_lse - ref_lse).max() <= LOSS_ATOL
    coef = np.array([1.0 / counts[p] for p, t in pairs])
    ref_dh = sco.rows_dh(hr, inp.W, yr, coef)
    got_dh = np.stack([dh[p, t] for p, t in pairs])
    assert rel_l2(got_dh, ref_dh) <= GRAD_RL2
    for i in range(len(pairs)):
        assert rel_l2(got_dh[i], ref_dh[i]) <= 2 * GRAD_RL2, pairs[i]
    # invalid rows are zero; the pass losses are the normalised sums of the row losses
    assert np.all(rows[idx < 0] == 0) and np.all(dh[idx < 0] == 0)
    for p in range(P):
        assert loss[p] == pytest.approx(rows[p].astype(np.float64).sum() / counts[p], rel=1e-5)
    assert loss[P] == pytest.approx(loss[:P].sum(), rel=1e-6)
    # dz rows sum to zero over the vocabulary up to their bf16 rounding: so do dW's columns
    assert np.all(np.isfinite(dW))
    col_sum = np.abs(dW.astype(np.float64).sum(axis=0))
    col_abs = np.abs(dW.astype(np.float64)).sum(axis=0)
    assert np.all(col_sum <= 1e-2 * col_abs + 1e-12)
