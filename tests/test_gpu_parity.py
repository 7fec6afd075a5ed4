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


def _check(w, kv_heads=None, seqs=None, with_grad=True, scale=None):
    inp = ttt_inputs.make_inputs(w)
    gpu = parity.run_gpu(w, inp, with_grad=with_grad, scale=scale)
    m = parity.compare_full(w, inp, gpu, with_grad=with_grad, kv_heads=kv_heads, seqs=seqs, scale=scale)
    print(w.name, "scale", scale, m)
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
    (3, 4, 2, 64, [5, 0, 70, 0]),      # empty sequences, one of them last
    (2, 2, 1, 128, [0, 129, 0, 1]),
])
def test_packed_ragged(P, H, Hkv, D, lengths):
    """THD with lengths that are not multiples of the tiles (1, 3, 17, 129, 257, ...) and
    with empty sequences (equal consecutive cu_seqlens entries)."""
    _check(ttt_inputs.thd("ragged", lengths, P, H, Hkv, D, 1e4))


def _random_config(seed):
    """A seeded random packed configuration: 1-6 sequences of 0-400 tokens, P in 1..5,
    D in {64, 128}, GQA groups of 1-4 with 1-3 KV heads, theta in {1e4, 1e6}."""
    rng = np.random.default_rng(seed)
    nseq = int(rng.integers(1, 7))
    lengths = [int(x) for x in rng.integers(0, 401, nseq)]
    if sum(lengths) == 0:
        lengths[0] = 1
    Hkv = int(rng.integers(1, 4))
    H = Hkv * int(rng.integers(1, 5))
    return dict(lengths=lengths, P=int(rng.integers(1, 6)), H=H, Hkv=Hkv, D=int(rng.choice([64, 128])),
                theta=float(rng.choice([1e4, 1e6])))


@needs_cuda
@pytest.mark.parametrize("seed", range(8))
def test_random_configurations(seed):
    """Seeded random combinations of the packed layout's parameters, every element against
    the oracle (the explicit cases above pin the individual edges; this covers their
    combinations)."""
    c = _random_config(1000 + seed)
    _check(ttt_inputs.thd(f"random{seed}", c["lengths"], c["P"], c["H"], c["Hkv"], c["D"], c["theta"]))


@needs_cuda
@pytest.mark.parametrize("B,S,P,H,Hkv,D", [(2, 200, 3, 4, 4, 128), (3, 64, 5, 2, 1, 64), (1, 384, 2, 8, 2, 128)])
def test_dense_tails(B, S, P, H, Hkv, D):
    _check(ttt_inputs.dense("dense_tail", B, S, P, H, Hkv, D, 1e6))


@needs_cuda
@pytest.mark.parametrize("layout,D", [("dense", 128), ("dense", 64), ("thd", 128), ("thd", 64)])
def test_non_default_softmax_scale(layout, D):
    """ttt_attn_desc.softmax_scale != 0: the trunk forward, the branch keys and merge of
    its epilogue, the trunk backward and the branch backward all take the descriptor's
    scale instead of 1/sqrt(D).  0.37/sqrt(D) and 2.5/sqrt(D) (sharper rows, so the
    forward's running-max rescale of O is exercised too), forward and backward, every
    element against the oracle run with the same scale."""
    for factor in (0.37, 2.5):
        if layout == "dense":
            w = ttt_inputs.dense("scale", 2, 200, 3, 4, 2, D, 1e4)
        else:
            w = ttt_inputs.thd("scale_thd", [129, 1, 300, 64], 4, 4, 1, D, 1e6)
        _check(w, scale=factor / D ** 0.5)


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
    # both evaluate the rotation in double and round it to bf16 through fp32: equal except
    # where the exact value sits within a few double ulps of a bf16 rounding boundary
    dq_ = np.abs(parity.to64(qr) - qr_ref)
    dk_ = np.abs(parity.to64(kr) - kr_ref)
    print("rotated q~ / k~ elements that differ:", int(np.sum(dq_ > 0)), int(np.sum(dk_ > 0)), "of", dq_.size, dk_.size)
    assert np.sum(dq_ > 0) <= 2 and np.sum(dk_ > 0) <= 2
    assert np.max(dq_) <= 2.0 ** -7 * np.max(np.abs(qr_ref))


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


# ----------------------------------------------------------------------------- full size

@needs_cuda
def test_deep_ttt_8k_sampled_group():
    """B=1, S=8192, P=7, 32/8 heads, D=128: full tensors of KV head 3 (its 4 query heads
    and all 7 passes) against the oracle."""
    _check(ttt_inputs.workloads()["deep_ttt_8k"], kv_heads=[3])


@needs_cuda
def test_thd_packed_sampled_sequences():
    """16 packed sequences (T = 38 264): full tensors of sequences 5 (649 tokens) and
    4 (3696 tokens), KV head 2."""
    _check(ttt_inputs.workloads()["thd_packed"], kv_heads=[2], seqs=[4, 5])


# positions at the edges of the 64-row and 128-row tiles and of the sequence
EDGE_POSITIONS_32K = [0, 1, 63, 64, 127, 128, 129, 255, 256, 4095, 4096, 4097, 8191, 8192, 16383, 16384,
                      24575, 32639, 32640, 32703, 32704, 32766, 32767]


@needs_cuda
def test_long_32k_sampled_rows():
    """B=1, S=32768, P=5, 32/8 heads, D=128, inputs scaled by 0.5, against the oracle's
    per-row forms: outputs, lse and dQ of ~300 query rows (every pass at the tile-edge
    positions, plus seeded random rows); dK/dV of the last 130 trunk keys of two KV heads
    (they cross the 128- and 64-row tile edges at 32640 and 32704), computed over every
    query row that sees them; dK/dV of branch keys at tile edges across the sequence."""
    w = ttt_inputs.workloads()["long_32k"]
    inp = ttt_inputs.make_inputs(w)
    gpu = parity.run_gpu(w, inp, with_grad=True)
    # float32 copies hold the bf16 values exactly; the oracle widens the rows it uses
    q, k, v, do = (t.float().numpy() for t in (inp.q, inp.k, inp.v, inp.do))
    g = w.H // w.Hkv
    L = w.lengths[0]
    rng = np.random.default_rng(0)
    rows = [(p0, i, (7 * n + 3 * p0) % w.H) for n, i in enumerate(EDGE_POSITIONS_32K) for p0 in range(w.P)]
    rows += [(int(rng.integers(w.P)), int(rng.integers(L)), int(rng.integers(w.H))) for _ in range(185)]
    kts = {}
    o_err, l_err = 0.0, 0.0
    dq_ref, dq_got = [[] for _ in range(w.P)], [[] for _ in range(w.P)]
    for (p0, i, h) in rows:
        kv = h // g
        if kv not in kts:
            kts[kv] = orc.rotate_trunk_keys(k, kv, w.theta)
        o_r, l_r = orc.row_forward(q, k, v, w.theta, p0, i, h, kt=kts[kv])
        o_err = max(o_err, float(np.max(np.abs(parity.to64(gpu["o"][p0, i, h]) - o_r))))
        l_err = max(l_err, abs(float(gpu["lse"][p0, 0, h, i]) - l_r))
        dq_ref[p0].append(orc.row_dq(q, k, v, do, w.theta, p0, i, h, kt=kts[kv]))
        dq_got[p0].append(parity.to64(gpu["dq"][p0, i, h]))
    t0 = L - 130
    dk_ref, dk_got, dv_ref, dv_got = [], [], [], []
    for kv in (0, 5):
        dk_t, dv_t = orc.tail_trunk_dkv(q, k, v, do, w.theta, kv, t0)
        dk_ref.append(dk_t)
        dv_ref.append(dv_t)
        dk_got.append(parity.to64(gpu["dk"][0, t0:, kv]))
        dv_got.append(parity.to64(gpu["dv"][0, t0:, kv]))
    bk_ref, bk_got, bv_ref, bv_got = [], [], [], []
    for (j0, t, kv) in [(1, 0, 2), (4, 127, 1), (2, 128, 7), (3, 4095, 4), (1, 4096, 6), (2, 9000, 7),
                        (4, 16384, 3), (3, 32703, 0), (1, 32767, 5), (4, 32767, 1)]:
        dk_r, dv_r = orc.row_dkv(q, k, v, do, w.theta, j0, t, kv)
        bk_ref.append(dk_r)
        bv_ref.append(dv_r)
        bk_got.append(parity.to64(gpu["dk"][j0, t, kv]))
        bv_got.append(parity.to64(gpu["dv"][j0, t, kv]))
    rel = lambda a_, b_: parity.rel_l2(np.array(a_), np.array(b_))
    dq_pass = [rel(dq_got[p], dq_ref[p]) for p in range(w.P) if dq_ref[p]]
    m = {"rows": len(rows), "o_max_abs": o_err, "lse_max_abs": l_err,
         "dq_rel_l2": rel(sum(dq_got, []), sum(dq_ref, [])), "dq_rel_l2_per_pass": dq_pass,
         "dk_rel_l2": rel(dk_got, dk_ref), "dv_rel_l2": rel(dv_got, dv_ref),
         "branch_dk_rel_l2": rel(bk_got, bk_ref), "branch_dv_rel_l2": rel(bv_got, bv_ref)}
    print("long_32k", m)
    parity.assert_within(m)
    assert m["branch_dk_rel_l2"] <= parity.GRAD_REL_L2 and m["branch_dv_rel_l2"] <= parity.GRAD_REL_L2, m


@needs_cuda
def test_long_32k_outputs_finite():
    """Whole-tensor property at the largest size: every output and lse entry is finite."""
    w = ttt_inputs.workloads()["long_32k"]
    inp = ttt_inputs.make_inputs(w, with_grad=False)
    gpu = parity.run_gpu(w, inp, with_grad=False)
    assert torch.isfinite(gpu["o"].float()).all()
    assert torch.isfinite(gpu["lse"]).all()


# ----------------------------------------------------------------------------- per-pass strides

def _pass_slots(t: torch.Tensor, pad: int) -> torch.Tensor:
    """Each pass written into its own slot of one larger buffer, slots `pad` elements apart
    beyond a packed pass: what a caller that produces the passes one at a time does
    instead of concatenating them."""
    P = t.shape[0]
    per = t[0].numel()
    buf = torch.full(((P - 1) * (per + pad) + per,), float("nan"), dtype=t.dtype, device=t.device)
    view = buf.as_strided(t.shape, (per + pad,) + t[0].stride())
    for p in range(P):
        view[p].copy_(t[p])
    return view


@needs_cuda
@pytest.mark.parametrize("layout", ["dense", "thd"])
def test_pass_strided_inputs(layout):
    """pass_stride_q / pass_stride_kv: q, k, v, dO with their passes at a padded common
    stride (different for the q and the kv kind), outputs allocated at the same strides.
    Against the oracle, and o, lse, dk, dv bit-identical to the packed call (same kernels;
    dq sums its fp32 partials in an unfixed order); the padding is never written."""
    from attention_pass_rope_b200 import ops
    if layout == "dense":
        w = ttt_inputs.dense("strided", 2, 200, 3, 4, 2, 128, 1e4)
    else:
        w = ttt_inputs.thd("strided_thd", [129, 1, 300, 64], 4, 8, 2, 64, 1e6)
    inp = ttt_inputs.make_inputs(w)
    q, k, v, do, cu = parity.gpu_shapes(w, inp)
    kw = dict(theta=w.theta, cu_seqlens=cu, max_seqlen=None if w.dense else w.max_seqlen)
    qs, dos = _pass_slots(q, 8 * 37), _pass_slots(do, 8 * 37)
    ks, vs = _pass_slots(k, 8 * 5), _pass_slots(v, 8 * 5)
    assert not qs.is_contiguous() and not ks.is_contiguous()
    o, lse = ops.ttt_attn_fwd(qs, ks, vs, **kw)
    dq, dk, dv = ops.ttt_attn_bwd(qs, ks, vs, o, lse, dos, **kw)
    torch.cuda.synchronize()
    assert o.stride(0) == qs.stride(0) and dq.stride(0) == qs.stride(0) and dk.stride(0) == ks.stride(0)
    gpu = {"o": parity.flat(o, w), "lse": lse, "dq": parity.flat(dq, w), "dk": parity.flat(dk, w),
           "dv": parity.flat(dv, w)}
    m = parity.compare_full(w, inp, gpu)
    print(layout, "strided", m)
    parity.assert_within(m)
    o_ref, lse_ref = ops.ttt_attn_fwd(q, k, v, **kw)
    _, dk_ref, dv_ref = ops.ttt_attn_bwd(q, k, v, o_ref, lse_ref, do, **kw)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
    assert torch.equal(dk, dk_ref) and torch.equal(dv, dv_ref)
    # the inputs' padding is untouched (still NaN) and nothing was read from it
    per = qs[0].numel()
    gap = qs.as_strided((qs.shape[0] - 1, qs.stride(0) - per), (qs.stride(0), 1), per)
    assert torch.isnan(gap.float()).all()


# ----------------------------------------------------------------------------- reuse of the rotation

@needs_cuda
@pytest.mark.parametrize("name", ["tiny", "ragged"])
def test_backward_reusing_forward_rotation(name):
    """TTT_FLAG_ROTATED_IN_WORKSPACE: one workspace for forward and backward, the backward
    skips the rotation.  Against the oracle, and dk/dv bit-identical to the path that
    rotates again (the rotation is deterministic; dq~ sums in an unfixed order)."""
    w = ttt_inputs.workloads()["tiny"] if name == "tiny" else \
        ttt_inputs.thd("ragged", [300, 128, 17, 1], 4, 8, 2, 128, 1e4)
    inp = ttt_inputs.make_inputs(w)
    gpu = parity.run_gpu(w, inp, reuse_rotation=True)
    m = parity.compare_full(w, inp, gpu)
    print(name, m)
    parity.assert_within(m)
    ref = parity.run_gpu(w, inp)
    assert torch.equal(gpu["dk"], ref["dk"]) and torch.equal(gpu["dv"], ref["dv"])
    assert torch.equal(gpu["o"], ref["o"]) and torch.equal(gpu["lse"], ref["lse"])


@needs_cuda
@pytest.mark.parametrize("name", ["tiny", "ragged"])
def test_forward_zeroes_backward_accumulator(name):
    """A forward given a backward-sized workspace zeroes the dq~ accumulator there and
    sets the mark after the status word; the backward that reuses the workspace skips
    its own zeroing and clears the mark, so a second backward on the same workspace
    zeroes again: same dk/dv bit for bit and the same dq up to the order of the fp32
    additions.  A forward-sized workspace gets no mark."""
    from attention_pass_rope_b200 import ops, ttt_attn_bwd, ttt_attn_fwd
    w = ttt_inputs.workloads()["tiny"] if name == "tiny" else \
        ttt_inputs.thd("ragged", [300, 128, 17, 1], 4, 8, 2, 128, 1e4)
    inp = ttt_inputs.make_inputs(w)
    q, k, v, do, cu = parity.gpu_shapes(w, inp)
    kw = dict(theta=w.theta, cu_seqlens=cu, max_seqlen=None if w.dense else w.max_seqlen)
    lay = ops._layout(q, k, v, cu, kw["max_seqlen"])
    mark = lambda ws: int(ws[4:8].view(torch.int32).item())  # noqa: E731
    ws = ops.alloc_workspace(ops.workspace_bytes(lay, w.theta, for_backward=True), q.device)
    ws.fill_(0xAB)  # the accumulator starts as garbage
    o, lse = ttt_attn_fwd(q, k, v, workspace=ws, **kw)
    torch.cuda.synchronize()
    assert mark(ws) == 0x01010101
    g1 = ttt_attn_bwd(q, k, v, o, lse, do, workspace=ws, rotated_in_workspace=True, **kw)
    torch.cuda.synchronize()
    assert mark(ws) == 0
    g2 = ttt_attn_bwd(q, k, v, o, lse, do, workspace=ws, rotated_in_workspace=True, **kw)
    torch.cuda.synchronize()
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])
    rel = float((g1[0].float() - g2[0].float()).norm() / g1[0].float().norm())
    assert rel < 1e-3, rel
    m = parity.compare_full(w, inp, {"o": parity.flat(o, w), "lse": lse, "dq": parity.flat(g1[0], w),
                                     "dk": parity.flat(g1[1], w), "dv": parity.flat(g1[2], w)})
    parity.assert_within(m)
    wsf = ops.alloc_workspace(ops.workspace_bytes(lay, w.theta, for_backward=False), q.device)
    wsf.fill_(0xAB)
    ttt_attn_fwd(q, k, v, workspace=wsf, **kw)
    torch.cuda.synchronize()
    assert mark(wsf) == 0


@needs_cuda
@pytest.mark.parametrize("keep_rotated", [False, True])
def test_autograd_function(keep_rotated):
    """ttt_attention under torch.autograd (both settings of keep_rotated) against the oracle."""
    from attention_pass_rope_b200 import ops
    w = ttt_inputs.workloads()["tiny"]
    inp = ttt_inputs.make_inputs(w)
    q, k, v, do, _ = parity.gpu_shapes(w, inp)
    q, k, v = (t.clone().requires_grad_(True) for t in (q, k, v))
    o = ops.ttt_attention(q, k, v, theta=w.theta, keep_rotated=keep_rotated)
    o.backward(do)
    torch.cuda.synchronize()
    gpu = {"o": parity.flat(o.detach(), w), "lse": ops.ttt_attn_fwd(q.detach(), k.detach(), v.detach(),
                                                                       theta=w.theta)[1],
           "dq": parity.flat(q.grad, w), "dk": parity.flat(k.grad, w), "dv": parity.flat(v.grad, w)}
    m = parity.compare_full(w, inp, gpu)
    print("autograd", keep_rotated, m)
    parity.assert_within(m)


# ----------------------------------------------------------------------------- maximum pass count

@needs_cuda
@pytest.mark.parametrize("layout,D", [("dense", 128), ("dense", 64), ("thd", 128)])
def test_sixteen_passes(layout, D):
    """P = 16, the largest pass count the library takes: 15 branch keys per query in the
    forward epilogue and 15 branch passes in the branch backward (its largest shared-memory
    layout), every output element against the oracle."""
    if layout == "dense":
        w = ttt_inputs.dense("p16", 1, 130, 16, 4, 2, D, 1e4)
    else:
        w = ttt_inputs.thd("p16_thd", [70, 1, 129], 16, 4, 1, D, 1e4)
    _check(w)


# ----------------------------------------------------------------------------- deterministic dq

@needs_cuda
@pytest.mark.parametrize("name", ["ragged", "4k"])
def test_deterministic_dq(name):
    """TTT_FLAG_DETERMINISTIC_DQ: the backward run twice gives bit-identical dq (and dk,
    dv), within the oracle's tolerance; on the 4K workload the oracle checks KV head 5."""
    from attention_pass_rope_b200 import ops
    if name == "ragged":
        w, kv = ttt_inputs.thd("ragged", [300, 128, 17, 1, 257], 3, 8, 2, 128, 1e4), None
    else:
        w, kv = ttt_inputs.workloads()["qwen3_8b_4k"], [5]
    inp = ttt_inputs.make_inputs(w)
    q, k, v, do, cu = parity.gpu_shapes(w, inp)
    kw = dict(theta=w.theta, cu_seqlens=cu, max_seqlen=None if w.dense else w.max_seqlen)
    o, lse = ops.ttt_attn_fwd(q, k, v, **kw)
    runs = [ops.ttt_attn_bwd(q, k, v, o, lse, do, deterministic=True, **kw) for _ in range(2)]
    torch.cuda.synchronize()
    for a_, b_ in zip(*runs):
        assert torch.equal(a_, b_)
    dq, dk, dv = runs[0]
    gpu = {"o": parity.flat(o, w), "lse": lse, "dq": parity.flat(dq, w), "dk": parity.flat(dk, w),
           "dv": parity.flat(dv, w)}
    m = parity.compare_full(w, inp, gpu, kv_heads=kv)
    print(name, "deterministic", m)
    parity.assert_within(m)
