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
