"""Pins of the soft cross-entropy distillation oracle against what the mathematics and
library routines fix (no GPU).  Each test would fail for a plausible slip in the oracle:
a wrong teacher shift, a dropped normalisation, a missing term of the loss, a wrong sign
or a transposed operand in the gradients."""

import math

import numpy as np
import pytest
import scipy.special
import scipy.stats
import torch
import torch.nn.functional as F

from oracle import softce_oracle as sco


def _inputs(lengths=(5, 9, 1, 4), P=3, V=37, d=16, seed=0, scale=1.0):
    g = np.random.default_rng(seed)
    T = sum(lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)]).tolist()
    h = g.standard_normal((P, T, d)) * scale
    W = g.standard_normal((V, d)) * 0.5
    y = g.standard_normal((T, V)) * 2.0
    return h, W, y, cu


def test_counts_closed_form():
    """With every position counted, pass p of a sequence of length n has max(n - p + 1, 0)
    valid pairs; a masked teacher position removes exactly one pair of each pass that
    reaches it."""
    lengths = (5, 9, 1, 4, 2)
    cu = np.concatenate([[0], np.cumsum(lengths)]).tolist()
    P = 4
    idx = sco.teacher_index(cu, P)
    for p in range(1, P + 1):
        assert (idx[p - 1] >= 0).sum() == sum(max(n - p + 1, 0) for n in lengths)
    mask = np.ones(cu[-1], dtype=bool)
    mask[7] = False             # position 2 of the second sequence (starts at 5)
    idx_m = sco.teacher_index(cu, P, mask)
    for p in range(1, P + 1):
        # tokens 7, 6, 5 reach position 7 at passes 1, 2, 3; at pass 4 the token would be
        # 4, in the first sequence, so that pass loses nothing
        lost = 1 if p <= 3 else 0
        assert (idx_m[p - 1] >= 0).sum() == (idx[p - 1] >= 0).sum() - lost
    assert not np.any(idx_m == 7)


def test_teacher_never_crosses_a_sequence():
    lengths = (3, 6, 2)
    cu = [0, 3, 9, 11]
    idx = sco.teacher_index(cu, 5)
    for s in range(3):
        seg = idx[:, cu[s]:cu[s + 1]]
        ok = seg[seg >= 0]
        assert np.all((ok >= cu[s]) & (ok < cu[s + 1]))


def test_one_hot_teacher_is_cross_entropy_per_pass():
    """A teacher peaked far above the rest is a hard label: each pass's loss is torch's
    mean cross-entropy over its valid pairs, the label of pair (p, t) being the token at
    teacher position t + p - 1 of its sequence."""
    lengths = (6, 3, 8)
    cu = np.concatenate([[0], np.cumsum(lengths)]).tolist()
    P, V, d = 3, 29, 12
    g = np.random.default_rng(3)
    T = cu[-1]
    h = g.standard_normal((P, T, d))
    W = g.standard_normal((V, d))
    tokens = g.integers(0, V, T)
    y = np.zeros((T, V))
    y[np.arange(T), tokens] = 200.0          # exp(-200) vanishes next to 1 in fp64
    out = sco.forward(h, W, y, cu)
    z = torch.from_numpy(h @ W.T)
    for p in range(1, P + 1):
        labels = torch.full((T,), -100, dtype=torch.long)
        for s in range(len(lengths)):
            for t in range(cu[s], cu[s + 1] - p + 1):
                labels[t] = int(tokens[t + p - 1])
        ref = F.cross_entropy(z[p - 1], labels, ignore_index=-100, reduction="mean").item()
        assert out["pass_loss"][p - 1] == pytest.approx(ref, rel=1e-12, abs=1e-12)
    assert out["loss"] == pytest.approx(out["pass_loss"].sum(), rel=1e-14)


def test_aligned_draft_has_near_zero_loss():
    """A draft whose logits peak at the token its teacher row names: loss ~ 0 when the
    teacher shift is right, about the logit gap when it is off by one."""
    lengths = (7, 5)
    cu = [0, 7, 12]
    P, V = 3, 11
    T = 12
    g = np.random.default_rng(5)
    tokens = g.integers(0, V, T)
    W = 40.0 * np.eye(V)
    y = np.full((T, V), -40.0)
    y[np.arange(T), tokens] = 40.0
    h = np.zeros((P, T, V))
    for s in range(2):
        for p in range(1, P + 1):
            for t in range(cu[s], cu[s + 1]):
                u = min(t + p - 1, cu[s + 1] - 1)
                h[p - 1, t, tokens[u]] = 1.0
    rows = sco.forward(h, W, y, cu)["rows"]
    assert np.max(rows) < 1e-12
    # the same draft against a teacher moved by one position pays the full gap
    y_shift = np.roll(y, 1, axis=0)
    rows_bad = sco.forward(h, W, y_shift, cu)["rows"]
    same = np.roll(tokens, 1) == tokens
    idx = sco.teacher_index(cu, P)
    bad = [(p, t) for p in range(P) for t in range(T) if idx[p, t] >= 0 and not same[idx[p, t]]]
    assert bad and min(rows_bad[p, t] for p, t in bad) > 30.0


def test_teacher_equal_to_student_gives_the_entropy():
    """q = softmax(z): the soft cross-entropy is the entropy of softmax(z) (scipy)."""
    h, W, y, cu = _inputs(P=1)
    z = h[0] @ W.T
    rows = sco.forward(h, W, z.copy(), cu)["rows"][0]
    for t in range(z.shape[0]):
        ent = scipy.stats.entropy(scipy.special.softmax(z[t]))
        assert rows[t] == pytest.approx(ent, rel=1e-12, abs=1e-13)


def test_uniform_draft_closed_form():
    """W = 0 makes every draft distribution uniform: l = log V for any teacher, so
    L_p = w_p * log V with local counts and w_p * n_p / N_p * log V with given counts."""
    h, W, y, cu = _inputs()
    V = W.shape[0]
    W0 = np.zeros_like(W)
    w = np.array([1.0, 0.5, 0.25])
    out = sco.forward(h, W0, y, cu, pass_weight=w)
    assert np.allclose(out["pass_loss"], w * math.log(V), rtol=1e-14)
    given = np.array([100.0, 80.0, 60.0])
    n = out["counts"]
    out_g = sco.forward(h, W0, y, cu, pass_weight=w, counts=given)
    assert np.allclose(out_g["pass_loss"], w * n / given * math.log(V), rtol=1e-14)
    # a pass with no valid pair contributes 0 (one-token sequences only, P = 2)
    out_e = sco.forward(h[:2, :1], W0, y[:1], [0, 1])
    assert out_e["pass_loss"][1] == 0.0


def test_shift_invariances():
    """Adding one vector to every vocabulary row of W shifts each row's logits by a
    constant; adding a constant to a teacher row leaves q unchanged: the loss keeps."""
    h, W, y, cu = _inputs(seed=7)
    base = sco.forward(h, W, y, cu)
    b = np.random.default_rng(8).standard_normal(W.shape[1])
    moved = sco.forward(h, W + b[None, :], y + 3.0, cu)
    assert np.allclose(moved["rows"], base["rows"], rtol=1e-10, atol=1e-11)
    # but a shift of one vocabulary entry's teacher logit does change it
    y2 = y.copy()
    y2[:, 0] += 1.0
    assert not np.allclose(sco.forward(h, W, y2, cu)["rows"], base["rows"])


def test_gradients_match_central_differences():
    h, W, y, cu = _inputs(lengths=(4, 3), P=2, V=9, d=5, seed=11)
    w = [1.0, 0.7]
    grad = 1.3
    dh, dW = sco.backward(h, W, y, cu, pass_weight=w, grad=grad)

    def loss(hh, WW):
        return grad * sco.forward(hh, WW, y, cu, pass_weight=w)["loss"]

    eps = 1e-6
    for (p, t, j) in [(0, 0, 0), (0, 3, 4), (1, 2, 1), (1, 5, 3), (0, 6, 2)]:
        hp, hm = h.copy(), h.copy()
        hp[p, t, j] += eps
        hm[p, t, j] -= eps
        fd = (loss(hp, W) - loss(hm, W)) / (2 * eps)
        assert dh[p, t, j] == pytest.approx(fd, rel=1e-6, abs=1e-9)
    for (v, j) in [(0, 0), (3, 4), (8, 2), (5, 1)]:
        Wp, Wm = W.copy(), W.copy()
        Wp[v, j] += eps
        Wm[v, j] -= eps
        fd = (loss(h, Wp) - loss(h, Wm)) / (2 * eps)
        assert dW[v, j] == pytest.approx(fd, rel=1e-6, abs=1e-9)
    # an invalid pair (the last token of a sequence at pass 2) has no gradient
    assert np.all(dh[1, 3] == 0) and np.all(dh[1, 6] == 0)


def test_gradient_invariants():
    """Each pair's logit gradient sums to zero over the vocabulary (softmax minus a
    distribution), so the columns of dW sum to zero; dh is W^T of it."""
    h, W, y, cu = _inputs(seed=13)
    dz = sco.logit_grad(h, W, y, cu)
    assert np.allclose(dz.sum(axis=-1), 0.0, atol=1e-15)
    dh, dW = sco.backward(h, W, y, cu)
    assert np.allclose(dW.sum(axis=0), 0.0, atol=1e-13)
    assert np.allclose(dh, np.einsum("ptv,vd->ptd", dz, W), rtol=1e-13, atol=1e-15)


def test_row_forms_match_the_full_forms():
    h, W, y, cu = _inputs(seed=17)
    out = sco.forward(h, W, y, cu, pass_weight=[1.0, 0.5, 2.0])
    dh, _ = sco.backward(h, W, y, cu, pass_weight=[1.0, 0.5, 2.0], grad=0.9)
    idx = sco.teacher_index(cu, 3)
    n = out["counts"]
    for (p, t) in [(0, 0), (1, 3), (2, 10), (0, 17)]:
        u = idx[p, t]
        assert u >= 0
        l, lse = sco.row_forward(h[p, t], W, y[u])
        assert l == pytest.approx(out["rows"][p, t], rel=1e-13)
        assert lse == pytest.approx(out["lse_z"][p, t], rel=1e-13)
        coef = 0.9 * [1.0, 0.5, 2.0][p] / n[p]
        assert np.allclose(sco.row_dh(h[p, t], W, y[u], coef), dh[p, t], rtol=1e-12, atol=1e-15)


def test_sliced_row_forms_match_the_full_forms():
    """The few-rows forms used at full size (vocabulary in slices) agree with the full
    forms, with a slice size that leaves a ragged last slice."""
    h, W, y, cu = _inputs(V=37, seed=19)
    w = [1.0, 0.5, 2.0]
    out = sco.forward(h, W, y, cu, pass_weight=w)
    dh, _ = sco.backward(h, W, y, cu, pass_weight=w, grad=1.1)
    idx = sco.teacher_index(cu, 3)
    pairs = [(0, 2), (1, 7), (2, 15), (0, 18)]
    hr = np.stack([h[p, t] for p, t in pairs])
    yr = np.stack([y[idx[p, t]] for p, t in pairs])
    coef = np.array([1.1 * w[p] / out["counts"][p] for p, t in pairs])
    loss, lse = sco.rows_forward(hr, W, yr)
    assert np.allclose(loss, [out["rows"][p, t] for p, t in pairs], rtol=1e-13)
    assert np.allclose(lse, [out["lse_z"][p, t] for p, t in pairs], rtol=1e-13)
    assert np.allclose(sco.rows_logits(hr, W, slice_rows=10), hr @ W.T, rtol=1e-14)
    assert np.allclose(sco.rows_dh(hr, W, yr, coef, slice_rows=10), [dh[p, t] for p, t in pairs],
                       rtol=1e-12, atol=1e-15)


def test_general_form_reduces_to_the_pass_form():
    """The TTT passes written as explicit teacher positions and groups give the pass form's
    values, forward and backward."""
    h, W, y, cu = _inputs(seed=23)
    P, T, d = h.shape
    mask = np.random.default_rng(24).random(T) < 0.8
    w = [1.0, 0.6, 0.3]
    teacher, group = sco.ttt_mapping(cu, P)
    ref = sco.forward(h, W, y, cu, mask, w)
    got = sco.forward_mapped(h.reshape(P * T, d), W, y, teacher, group, P, mask, w)
    assert np.allclose(got["rows"], ref["rows"].reshape(-1), rtol=1e-13, atol=1e-15)
    assert np.allclose(got["group_loss"], ref["pass_loss"], rtol=1e-13)
    dh_ref, dW_ref = sco.backward(h, W, y, cu, mask, w, grad=0.7)
    dh, dW = sco.backward_mapped(h.reshape(P * T, d), W, y, teacher, group, P, mask, w, grad=0.7)
    assert np.allclose(dh, dh_ref.reshape(P * T, d), rtol=1e-12, atol=1e-15)
    assert np.allclose(dW, dW_ref, rtol=1e-12, atol=1e-15)


def test_per_slot_groups_closed_form_and_independence():
    """Block slots as groups: with W = 0 every valid row costs log V, so L_g = w_g log V for
    any slot with a valid row; a row's teacher outside [0, Ty) or masked is invalid; moving a
    row to another group changes only those two groups' losses."""
    g = np.random.default_rng(29)
    nb, Bs, d, V, Ty = 5, 4, 8, 13, 30
    R = nb * Bs
    h = g.standard_normal((R, d))
    y = g.standard_normal((Ty, V))
    anchors = np.array([0, 6, 11, 20, 28])
    teacher = np.array([a + j for a in anchors for j in range(Bs)])      # last block runs past Ty
    group = np.tile(np.arange(Bs), nb)
    mask = np.ones(Ty, dtype=bool)
    mask[7] = False
    out0 = sco.forward_mapped(h, np.zeros((V, d)), y, teacher, group, Bs, mask, [1.0, 2.0, 0.5, 0.25])
    valid = out0["valid"]
    assert not valid[teacher >= Ty].any() and not valid[teacher == 7].any()
    for s_ in range(Bs):
        if valid[group == s_].any():
            assert out0["group_loss"][s_] == pytest.approx([1.0, 2.0, 0.5, 0.25][s_] * math.log(V), rel=1e-13)
    W = g.standard_normal((V, d))
    base = sco.forward_mapped(h, W, y, teacher, group, Bs)
    g2 = group.copy()
    g2[5] = 3                                                            # row 5 (slot 1) moves to slot 3
    moved = sco.forward_mapped(h, W, y, teacher, g2, Bs)
    assert np.allclose(moved["group_loss"][[0, 2]], base["group_loss"][[0, 2]], rtol=1e-14)
    assert not np.isclose(moved["group_loss"][1], base["group_loss"][1])
    assert np.allclose(moved["rows"], base["rows"], rtol=1e-14)


def test_general_form_gradients_match_central_differences():
    g = np.random.default_rng(31)
    R, d, V, Ty, G = 7, 4, 6, 5, 3
    h = g.standard_normal((R, d))
    W = g.standard_normal((V, d))
    y = g.standard_normal((Ty, V))
    teacher = np.array([0, 1, 4, -1, 2, 9, 3])
    group = np.array([0, 1, 2, 0, 1, 2, 2])
    wts = [0.5, 1.5, 1.0]
    dh, dW = sco.backward_mapped(h, W, y, teacher, group, G, None, wts, grad=1.2)

    def L(hh, WW):
        return 1.2 * sco.forward_mapped(hh, WW, y, teacher, group, G, None, wts)["loss"]

    eps = 1e-6
    for (r, j) in [(0, 0), (2, 3), (4, 1), (6, 2)]:
        hp, hm = h.copy(), h.copy()
        hp[r, j] += eps
        hm[r, j] -= eps
        assert dh[r, j] == pytest.approx((L(hp, W) - L(hm, W)) / (2 * eps), rel=1e-6, abs=1e-9)
    for (v, j) in [(0, 0), (5, 3), (2, 1)]:
        Wp, Wm = W.copy(), W.copy()
        Wp[v, j] += eps
        Wm[v, j] -= eps
        assert dW[v, j] == pytest.approx((L(h, Wp) - L(h, Wm)) / (2 * eps), rel=1e-6, abs=1e-9)
    assert np.all(dh[3] == 0) and np.all(dh[5] == 0)                    # teacher -1 and past Ty


def test_oracle_matches_its_fixture():
    """The soft-CE oracle reproduces tests/golden/softce_fixture.txt (written by the
    committed tests/golden/make_softce_fixture.py, which calls the oracle only): any later
    change to the oracle's arithmetic shows up here.  The fixture's invalid rows (a masked
    teacher position, positions past a sequence's end or past the teacher rows) are 0."""
    import os
    import sys
    golden = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
    sys.path.insert(0, golden)
    import make_softce_fixture as mk
    ref = mk.read(os.path.join(golden, "softce_fixture.txt"))
    got = mk.compute()
    assert set(ref) == set(got)
    for name in ref:
        np.testing.assert_allclose(np.asarray(got[name]), ref[name], rtol=0, atol=1e-13, err_msg=name)
    assert ref["rows"][0, 3] == 0 and ref["rows"][1, 2] == 0 and ref["rows"][1, 4] == 0
    assert ref["g_rows"][3] == 0 and ref["g_rows"][5] == 0
