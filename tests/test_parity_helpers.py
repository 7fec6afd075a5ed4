"""CPU checks of the comparison helpers that the GPU parity tests rely on.  A planted
mistake lives in a copy of the oracle's own output, never in a kernel."""

import numpy as np
import pytest

import ttt_inputs
from oracle import ttt_oracle as orc
from tests import parity


def _oracle_grads(P=3, L=96):
    w = ttt_inputs.thd("helpers", [L], P, 4, 2, 64, 1e4)
    inp = ttt_inputs.make_inputs(w)
    q, k, v, do = parity.oracle_np(inp)
    O, lse = orc.forward_packed(q, k, v, w.cu_seqlens, w.theta, False)
    return w, orc.backward_packed(q, k, v, do, lse, w.cu_seqlens, w.theta, False)


def test_branch_pass_error_hidden_in_whole_tensor_is_caught_per_pass():
    """Pass 1 carries most of dK's norm (every trunk key), so a 3 % error confined to the
    branch passes stays under the whole-tensor bound; the per-pass figure exceeds it."""
    w, (dq, dk, dv) = _oracle_grads()
    bad = dk.copy()
    rng = np.random.default_rng(7)
    bad[1:] += 0.03 * np.linalg.norm(dk[1:]) / np.sqrt(dk[1:].size) * rng.standard_normal(dk[1:].shape)
    assert parity.rel_l2(bad, dk) <= parity.GRAD_REL_L2
    per_pass, worst = parity.per_pass_rel_l2(bad, dk)
    assert per_pass[0] == 0.0 and max(per_pass[1:]) > parity.GRAD_REL_L2
    assert worst[1][0] >= 1
    m = {"o_max_abs": 0.0, "lse_max_abs": 0.0, "dk_rel_l2": parity.rel_l2(bad, dk), "dk_rel_l2_per_pass": per_pass}
    with pytest.raises(AssertionError):
        parity.assert_within(m)


def test_per_pass_skips_unsampled_entries():
    """NaN entries of the reference (outside a sampled subset) are skipped, and a pass with
    no sampled entry reports None instead of failing."""
    ref = np.full((2, 5, 3, 4), np.nan)
    ref[0, :, 1] = 1.0
    got = np.zeros_like(ref)
    got[0, :, 1] = 1.0
    per_pass, worst = parity.per_pass_rel_l2(got, ref)
    assert per_pass == [0.0, None] and worst == (0.0, None)


def _block_oracle_as_gpu(w, inp):
    """The block oracle's own results laid out like the library's outputs."""
    import torch
    from oracle import block_draft_oracle as bd
    f64 = lambda x: x.float().numpy().astype(np.float64)
    out = {"o": np.zeros((w.NB, w.Bs, w.H, w.D)), "dqb": np.zeros((w.NB, w.Bs, w.H, w.D)),
           "dk_ctx": np.zeros((w.Tc, w.Hkv, w.D)), "dv_ctx": np.zeros((w.Tc, w.Hkv, w.D)),
           "dkb": np.zeros((w.NB, w.Bs, w.Hkv, w.D)), "dvb": np.zeros((w.NB, w.Bs, w.Hkv, w.D))}
    lse = np.zeros((w.nseq, w.H, w.nblocks[0] * w.Bs)) if w.dense else np.zeros((w.H, w.NB * w.Bs))
    for n in range(w.nseq):
        c0, c1, b0, b1 = w.cu_ctx[n], w.cu_ctx[n + 1], w.cu_blocks[n], w.cu_blocks[n + 1]
        if b1 == b0:
            continue
        c = dict(k_ctx=f64(inp.k_ctx[c0:c1]), v_ctx=f64(inp.v_ctx[c0:c1]), anchors=inp.anchors[b0:b1].tolist(),
                 qb=f64(inp.qb[b0:b1]), kb=f64(inp.kb[b0:b1]), vb=f64(inp.vb[b0:b1]))
        O, l = bd.forward_twopart(theta=w.theta, rope_round="bf16", **c)
        g = bd.backward_twopart(do=f64(inp.do[b0:b1]), O=O, lse=l, theta=w.theta, rope_round="bf16", **c)
        out["o"][b0:b1] = O
        rows = l.transpose(1, 0, 2).reshape(w.H, -1)
        if w.dense:
            lse[n] = rows
        else:
            lse[:, b0 * w.Bs:b1 * w.Bs] = rows
        out["dqb"][b0:b1], out["dk_ctx"][c0:c1], out["dv_ctx"][c0:c1], out["dkb"][b0:b1], out["dvb"][b0:b1] = g
    res = {k: torch.tensor(v) for k, v in out.items()}
    res["lse"] = torch.tensor(lse)
    return res


@pytest.mark.parametrize("dense", [True, False])
def test_block_compare_helper_reads_zero_on_the_oracle_and_flags_a_mistake(dense):
    import ttt_inputs
    from tests import block_parity as bp
    if dense:
        w = ttt_inputs.block_dense("h", 2, 40, 3, 4, 4, 2, 16, 1e4)
    else:
        w = ttt_inputs.block_thd("h", [1, 50, 0, 33], [1, 4, 0, 2], 5, 4, 2, 16, 1e4)
    inp = ttt_inputs.make_block_inputs(w)
    gpu = _block_oracle_as_gpu(w, inp)
    m = bp.compare(w, inp, gpu)
    assert max(v for k, v in m.items()) < 1e-6, m  # the helper widens through float32
    m = bp.compare(w, inp, gpu, kv_heads=[1], seqs=[1])
    assert max(v for k, v in m.items()) < 1e-6, m  # the helper widens through float32
    gpu["dk_ctx"] = gpu["dk_ctx"] * 1.03
    with pytest.raises(AssertionError):
        bp.assert_within(bp.compare(w, inp, gpu))
