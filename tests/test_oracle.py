"""Pins for the fp64 oracle: everything here checks it against something other
than itself (a second formulation, a library routine, finite differences,
closed forms and invariants).  CPU only."""

import math
import os
import sys

import numpy as np
import pytest
import torch

from oracle import ttt_oracle as orc

RNG = np.random.default_rng(1234)


def rnd(*shape):
    return RNG.standard_normal(shape)


def rope_complex(x, pos, theta):
    """Independent RoPE: pair (d, d + D/2) as the complex number x_d + i x_{d+D/2},
    multiplied by exp(i * pos * theta**(-2d/D))."""
    D = x.shape[-1]
    z = x[..., : D // 2] + 1j * x[..., D // 2:]
    freq = np.array([theta ** (-2.0 * d / D) for d in range(D // 2)])
    w = np.exp(1j * np.asarray(pos, dtype=np.float64)[:, None] * freq[None, :])
    z = z * w.reshape((len(pos),) + (1,) * (z.ndim - 2) + (D // 2,))
    return np.concatenate([z.real, z.imag], axis=-1)


# ---------------------------------------------------------------- bf16 rounding

def test_bf16_round_special_values():
    one = 1.0
    assert orc.bf16_round(np.array([one]))[0] == 1.0
    # halfway between 1 and 1+2^-7: ties to even -> 1
    assert orc.bf16_round(np.array([1.0 + 2.0 ** -8]))[0] == 1.0
    # halfway between 1+2^-7 and 1+2^-6: ties to even -> 1+2^-6
    assert orc.bf16_round(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6
    # just above halfway rounds up
    assert orc.bf16_round(np.array([1.0 + 2.0 ** -8 + 2.0 ** -20]))[0] == 1.0 + 2.0 ** -7
    assert orc.bf16_round(np.array([-3.0]))[0] == -3.0


def test_bf16_round_matches_torch_cast():
    x = (RNG.standard_normal(200000) * np.exp(RNG.uniform(-20, 20, 200000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(orc.bf16_round(x.astype(np.float64)), ref)


# ---------------------------------------------------------------- RoPE

def test_rope_matches_complex_rotation():
    x = rnd(9, 3, 16)
    pos = np.arange(9) * 37 + 5
    np.testing.assert_allclose(orc.rope_rotate(x, pos, 1e4), rope_complex(x, pos, 1e4), atol=1e-12)


def test_rope_relative_shift_identity():
    """R(m)x . R(n)y = x . R(n-m)y: the score depends on the position difference only."""
    D = 64
    for m, n in [(0, 0), (3, 11), (4095, 7), (1000, 32767)]:
        x, y = rnd(1, 1, D), rnd(1, 1, D)
        lhs = np.sum(orc.rope_rotate(x, [m], 1e6) * orc.rope_rotate(y, [n], 1e6))
        rhs = np.sum(x * orc.rope_rotate(y, [n - m], 1e6))
        assert abs(lhs - rhs) < 1e-10 * (1 + abs(lhs))


def test_rope_inverse_is_adjoint():
    x, y = rnd(7, 2, 32), rnd(7, 2, 32)
    pos = np.arange(7) + 100
    np.testing.assert_allclose(orc.rope_rotate(orc.rope_rotate(x, pos, 1e4), pos, 1e4, inverse=True), x,
                               atol=1e-12)
    lhs = np.sum(orc.rope_rotate(x, pos, 1e4) * y)
    rhs = np.sum(x * orc.rope_rotate(y, pos, 1e4, inverse=True))
    assert abs(lhs - rhs) < 1e-10


def test_pass_offsets_pin_scores():
    """Trunk score of (pass p, position i) vs trunk key t depends on (i+p-1)-t; branch
    score vs pass-j key at position i on p-j (checked with the complex rotation)."""
    P, L, D, theta = 4, 6, 16, 1e4
    q, k = rnd(P, L, 1, D), rnd(P, L, 1, D)
    qr, kr = orc.rotate_inputs(q, k, theta, rope_round=None)
    for p in range(P):          # 0-based pass index; 1-based pass p+1 -> offset p
        for i in range(L):
            for t in range(i + 1):
                ref = np.sum(q[p, i, 0] * rope_complex(k[0, t:t + 1, :], [t - (i + p)], theta)[0, 0])
                assert abs(np.sum(qr[p, i, 0] * kr[0, t, 0]) - ref) < 1e-10
            for j in range(1, p + 1):
                ref = np.sum(q[p, i, 0] * rope_complex(k[j, i:i + 1, :], [j - p], theta)[0, 0])
                assert abs(np.sum(qr[p, i, 0] * kr[j, i, 0]) - ref) < 1e-10


# ---------------------------------------------------------------- staircase

def test_staircase_key_counts():
    P, L = 5, 9
    m = orc.staircase_mask(P, L)
    counts = m.sum(axis=1).reshape(P, L)
    for p in range(P):
        for i in range(L):
            assert counts[p, i] == (i + 1) + p


@pytest.mark.parametrize("P,L,H,Hkv,D", [(1, 5, 2, 1, 8), (3, 7, 4, 2, 16), (4, 17, 2, 2, 8), (2, 1, 3, 1, 4)])
@pytest.mark.parametrize("rope_round", [None, "bf16"])
def test_twopart_equals_bruteforce_forward(P, L, H, Hkv, D, rope_round):
    q, k, v = rnd(P, L, H, D), rnd(P, L, Hkv, D), rnd(P, L, Hkv, D)
    O1, l1 = orc.forward_bruteforce(q, k, v, 1e4, rope_round=rope_round)
    O2, l2 = orc.forward_twopart(q, k, v, 1e4, rope_round=rope_round, block=4)
    np.testing.assert_allclose(O2, O1, atol=1e-13)
    np.testing.assert_allclose(l2, l1, atol=1e-13)


@pytest.mark.parametrize("P,L,H,Hkv,D", [(1, 5, 2, 1, 8), (3, 7, 4, 2, 16), (4, 17, 2, 2, 8)])
def test_twopart_equals_bruteforce_backward(P, L, H, Hkv, D):
    q, k, v, do = rnd(P, L, H, D), rnd(P, L, Hkv, D), rnd(P, L, Hkv, D), rnd(P, L, H, D)
    _, lse = orc.forward_twopart(q, k, v, 1e4)
    g1 = orc.backward_bruteforce(q, k, v, do, 1e4)
    g2 = orc.backward_twopart(q, k, v, do, lse, 1e4, block=5)
    for a, b in zip(g2, g1):
        np.testing.assert_allclose(a, b, atol=1e-12)


def test_merge_parts():
    """Pass 1 has an empty branch (lse_b = -inf, O = O_t); later passes satisfy
    lse = logaddexp(lse_t, lse_b)."""
    P, L, H, D = 3, 6, 2, 8
    q, k, v = rnd(P, L, H, D), rnd(P, L, 1, D), rnd(P, L, 1, D)
    O, lse, parts = orc.forward_twopart(q, k, v, 1e4, return_parts=True)
    assert np.all(np.isneginf(parts["lse_b"][0]))
    np.testing.assert_array_equal(O[0], parts["O_t"][0])
    np.testing.assert_array_equal(lse[0], parts["lse_t"][0])
    assert np.all(np.isfinite(O)) and np.all(np.isfinite(lse))
    assert np.all(lse[1:] > parts["lse_t"][1:])


# ---------------------------------------------------------------- library cross-checks

def torch_rope(x, pos, theta):
    D = x.shape[-1]
    freq = torch.tensor([theta ** (-2.0 * d / D) for d in range(D // 2)], dtype=torch.float64)
    ang = torch.tensor(pos, dtype=torch.float64)[:, None] * freq[None, :]
    z = torch.complex(x[..., : D // 2], x[..., D // 2:]) * torch.polar(torch.ones_like(ang), ang)[:, None, :]
    return torch.cat([z.real, z.imag], dim=-1)


def test_single_pass_equals_sdpa():
    """P = 1 reduces to causal GQA attention with RoPE at position i (torch SDPA, fp64)."""
    L, H, Hkv, D, theta = 11, 4, 2, 16, 1e4
    q, k, v, do = rnd(1, L, H, D), rnd(1, L, Hkv, D), rnd(1, L, Hkv, D), rnd(1, L, H, D)
    O, lse = orc.forward_twopart(q, k, v, theta, rope_round=None)
    dq, dk, dv = orc.backward_twopart(q, k, v, do, lse, theta, rope_round=None)

    tq = torch.tensor(q[0], requires_grad=True)
    tk = torch.tensor(k[0], requires_grad=True)
    tv = torch.tensor(v[0], requires_grad=True)
    pos = list(range(L))
    qr = torch_rope(tq, pos, theta).transpose(0, 1)                  # [H, L, D]
    kr = torch_rope(tk, pos, theta).transpose(0, 1).repeat_interleave(H // Hkv, 0)
    vv = tv.transpose(0, 1).repeat_interleave(H // Hkv, 0)
    out = torch.nn.functional.scaled_dot_product_attention(qr[None], kr[None], vv[None], is_causal=True)[0]
    out = out.transpose(0, 1)
    np.testing.assert_allclose(O[0], out.detach().numpy(), atol=1e-12)
    (out * torch.tensor(do[0])).sum().backward()
    np.testing.assert_allclose(dq[0], tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk[0], tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv[0], tv.grad.numpy(), atol=1e-11)


def test_finite_differences():
    """Central differences of sum(O * dO) (exact RoPE) against the analytic gradients."""
    P, L, H, Hkv, D, theta = 3, 4, 2, 1, 8, 1e4
    q, k, v, do = rnd(P, L, H, D), rnd(P, L, Hkv, D), rnd(P, L, Hkv, D), rnd(P, L, H, D)
    _, lse = orc.forward_twopart(q, k, v, theta, rope_round=None)
    grads = orc.backward_twopart(q, k, v, do, lse, theta, rope_round=None)

    def loss(q_, k_, v_):
        O, _ = orc.forward_bruteforce(q_, k_, v_, theta, rope_round=None)
        return float(np.sum(O * do))

    eps = 1e-6
    for which, arr in enumerate((q, k, v)):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            plus = [q.copy(), k.copy(), v.copy()]
            minus = [q.copy(), k.copy(), v.copy()]
            plus[which][idx] += eps
            minus[which][idx] -= eps
            fd[idx] = (loss(*plus) - loss(*minus)) / (2 * eps)
        np.testing.assert_allclose(grads[which], fd, atol=2e-8)


# ---------------------------------------------------------------- invariants

def test_position_shift_invariance():
    """Adding a constant to every position leaves outputs and gradients unchanged."""
    P, L, H, D, theta = 3, 9, 2, 16, 1e4
    q, k, v, do = rnd(P, L, H, D), rnd(P, L, 1, D), rnd(P, L, 1, D), rnd(P, L, H, D)
    O0, l0 = orc.forward_twopart(q, k, v, theta, rope_round=None)
    O1, l1 = orc.forward_twopart(q, k, v, theta, rope_round=None, pos_offset=123)
    np.testing.assert_allclose(O1, O0, atol=1e-12)
    np.testing.assert_allclose(l1, l0, atol=1e-12)
    g0 = orc.backward_twopart(q, k, v, do, l0, theta, rope_round=None)
    g1 = orc.backward_twopart(q, k, v, do, l1, theta, rope_round=None, pos_offset=123)
    # scores depend on position differences only, so O is the same function of the
    # pre-RoPE inputs for every offset, and so are its gradients
    for a, b in zip(g1, g0):
        np.testing.assert_allclose(a, b, atol=1e-11)


def test_single_key():
    """i = 0 at pass 1: the only visible key is trunk key 0: O = V_1[0], lse = s."""
    D = 8
    q, k, v = rnd(1, 1, 1, D), rnd(1, 1, 1, D), rnd(1, 1, 1, D)
    O, lse = orc.forward_twopart(q, k, v, 1e4, rope_round=None)
    np.testing.assert_allclose(O[0, 0, 0], v[0, 0, 0], atol=1e-15)
    # position 0 rotates by zero angle
    assert abs(lse[0, 0, 0] - np.dot(q[0, 0, 0], k[0, 0, 0]) / math.sqrt(D)) < 1e-14


def test_uniform_scores_average_values():
    """All scores equal (q = 0): O is the plain mean of the visible values, lse = log(count)."""
    P, L, D = 3, 5, 8
    q = np.zeros((P, L, 1, D))
    k, v = rnd(P, L, 1, D), rnd(P, L, 1, D)
    O, lse = orc.forward_twopart(q, k, v, 1e4, rope_round=None)
    for p in range(P):
        for i in range(L):
            vis = [v[0, t, 0] for t in range(i + 1)] + [v[j, i, 0] for j in range(1, p + 1)]
            np.testing.assert_allclose(O[p, i, 0], np.mean(vis, axis=0), atol=1e-14)
            assert abs(lse[p, 0, i] - math.log(len(vis))) < 1e-14


def test_packed_layouts():
    """Dense and THD packing: per-sequence results, lse in [P,B,H,S] / [P,H,T]."""
    P, H, Hkv, D = 2, 2, 1, 8
    lens = [5, 3, 7]
    T = sum(lens)
    cu = np.cumsum([0] + lens)
    q, k, v, do = rnd(P, T, H, D), rnd(P, T, Hkv, D), rnd(P, T, Hkv, D), rnd(P, T, H, D)
    O, lse = orc.forward_packed(q, k, v, cu, 1e4, dense=False)
    assert lse.shape == (P, H, T)
    for n in range(3):
        a, b = cu[n], cu[n + 1]
        Os, ls = orc.forward_twopart(q[:, a:b], k[:, a:b], v[:, a:b], 1e4)
        np.testing.assert_array_equal(O[:, a:b], Os)
        np.testing.assert_array_equal(lse[:, :, a:b], ls)
    dq, dk, dv = orc.backward_packed(q, k, v, do, lse, cu, 1e4, dense=False)
    g = orc.backward_twopart(q[:, 5:8], k[:, 5:8], v[:, 5:8], do[:, 5:8], lse[:, :, 5:8], 1e4)
    np.testing.assert_array_equal(dq[:, 5:8], g[0])
    # dense: equal lengths, lse [P, B, H, S]
    cu2 = np.array([0, 4, 8])
    O2, lse2 = orc.forward_packed(q[:, :8], k[:, :8], v[:, :8], cu2, 1e4, dense=True)
    assert lse2.shape == (P, 2, H, 4)
    Os, ls = orc.forward_twopart(q[:, 4:8], k[:, 4:8], v[:, 4:8], 1e4)
    np.testing.assert_array_equal(lse2[:, 1], ls)


def test_single_row_functions_match_full_oracle():
    """The per-row forms (used on samples of full-size workloads) agree with the
    two-part oracle element by element."""
    P, L, H, Hkv, D = 3, 9, 4, 2, 8
    q, k, v, do = rnd(P, L, H, D), rnd(P, L, Hkv, D), rnd(P, L, Hkv, D), rnd(P, L, H, D)
    O, lse = orc.forward_twopart(q, k, v, 1e4)
    dq, dk, dv = orc.backward_twopart(q, k, v, do, lse, 1e4)
    for (p0, i, h) in [(0, 0, 0), (1, 4, 3), (2, 8, 1), (2, 0, 2)]:
        o_r, l_r = orc.row_forward(q, k, v, 1e4, p0, i, h)
        np.testing.assert_allclose(o_r, O[p0, i, h], atol=1e-13)
        assert abs(l_r - lse[p0, h, i]) < 1e-13
        np.testing.assert_allclose(orc.row_dq(q, k, v, do, 1e4, p0, i, h), dq[p0, i, h], atol=1e-12)
    for (j0, t, kv) in [(0, 0, 0), (0, 7, 1), (1, 3, 0), (2, 8, 1)]:
        dk_r, dv_r = orc.row_dkv(q, k, v, do, 1e4, j0, t, kv)
        np.testing.assert_allclose(dk_r, dk[j0, t, kv], atol=1e-12)
        np.testing.assert_allclose(dv_r, dv[j0, t, kv], atol=1e-12)


@pytest.mark.parametrize("t0", [0, 5, 8])
def test_tail_trunk_dkv_matches_full_oracle(t0):
    """The vectorised gradient of the last trunk keys (used on 32K-token samples)
    agrees with the two-part oracle's full backward on every key t >= t0."""
    P, L, H, Hkv, D = 3, 9, 4, 2, 8
    q, k, v, do = rnd(P, L, H, D), rnd(P, L, Hkv, D), rnd(P, L, Hkv, D), rnd(P, L, H, D)
    O, lse = orc.forward_twopart(q, k, v, 1e4)
    dq, dk, dv = orc.backward_twopart(q, k, v, do, lse, 1e4)
    for kv in range(Hkv):
        dk_t, dv_t = orc.tail_trunk_dkv(q, k, v, do, 1e4, kv, t0)
        np.testing.assert_allclose(dk_t, dk[0, t0:, kv], atol=1e-12)
        np.testing.assert_allclose(dv_t, dv[0, t0:, kv], atol=1e-12)


def test_chunk_partial_whole_sequence_equals_the_oracle():
    """One chunk holding the whole sequence, with its branch keys, is the full attention."""
    P, L, H, Hkv, D = 3, 11, 4, 2, 8
    q, k, v = rnd(P, L, H, D), rnd(P, L, Hkv, D), rnd(P, L, Hkv, D)
    O, lse = orc.forward_twopart(q, k, v, 1e4)
    Oc, lc = orc.chunk_partial(q, k[0], v[0], 1e4, 0, 0, branch_k=k, branch_v=v)
    np.testing.assert_allclose(Oc, O, atol=1e-13)
    np.testing.assert_allclose(lc, lse, atol=1e-13)


@pytest.mark.parametrize("cuts", [(4, 7), (1, 10), (5,)])
def test_chunk_partials_merge_to_the_oracle(cuts):
    """Partials of every query chunk over every trunk-key chunk (its own chunk taking the
    branch keys), merged by log-sum-exp (written out here), equal the full attention;
    chunks that start after the query chunk contribute lse = -inf."""
    P, L, H, Hkv, D = 3, 11, 4, 2, 8
    q, k, v = rnd(P, L, H, D), rnd(P, L, Hkv, D), rnd(P, L, Hkv, D)
    O, lse = orc.forward_twopart(q, k, v, 1e4)
    bounds = [0, *cuts, L]
    for qa, qb in zip(bounds[:-1], bounds[1:]):
        acc_o, acc_l = None, None
        for ka, kb in zip(bounds[:-1], bounds[1:]):
            own = ka == qa
            Op, lp = orc.chunk_partial(q[:, qa:qb], k[0, ka:kb], v[0, ka:kb], 1e4, qa, ka,
                                       branch_k=k[:, qa:qb] if own else None, branch_v=v[:, qa:qb] if own else None)
            if ka > qa:
                assert np.all(lp == -np.inf) and np.all(Op == 0.0)
            if acc_o is None:
                acc_o, acc_l = Op, lp
                continue
            m = np.maximum(acc_l, lp)
            ms = np.where(np.isfinite(m), m, 0.0)
            l = ms + np.log(np.exp(acc_l - ms) + np.exp(lp - ms))
            wa = np.exp(acc_l - l).transpose(0, 2, 1)[..., None]
            wb = np.exp(lp - l).transpose(0, 2, 1)[..., None]
            acc_o, acc_l = wa * acc_o + wb * Op, l
        np.testing.assert_allclose(acc_o, O[:, qa:qb], atol=1e-12)
        np.testing.assert_allclose(acc_l, lse[:, :, qa:qb], atol=1e-12)


# ---------------------------------------------------------------- golden fixtures

def _golden(name):
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", name)


def test_staircase_rope_shift_machine_precision():
    """NeMo-RL PR 3725's self-review reports that the multi-pass staircase visibility and
    the RoPE-relative shift agree with an independent rotate-half oracle to machine
    precision in fp64 (the figure is in tests/golden/staircase_rope_shift_fp64.txt).  The
    oracle's two forms of the same function -- trunk + branch merged by log-sum-exp, and
    one softmax over the explicit staircase mask -- must agree to within a few times that
    figure on short sequences; a wrong shift, mask or merge term is off by orders of
    magnitude more."""
    with open(_golden("staircase_rope_shift_fp64.txt")) as f:
        bound = float([ln.split()[1] for ln in f if ln.startswith("max_abs_diff")][0])
    rng = np.random.default_rng(1)
    worst = 0.0
    for P, L, H, Hkv, D in [(1, 5, 2, 1, 8), (3, 7, 4, 2, 16), (4, 17, 2, 2, 8), (2, 1, 3, 1, 4)]:
        q, k, v = (rng.standard_normal(s) for s in ((P, L, H, D), (P, L, Hkv, D), (P, L, Hkv, D)))
        O1, l1 = orc.forward_bruteforce(q, k, v, 1e4, rope_round=None)
        O2, l2 = orc.forward_twopart(q, k, v, 1e4, rope_round=None, block=4)
        worst = max(worst, float(np.max(np.abs(O2 - O1))), float(np.max(np.abs(l2 - l1))))
    assert worst <= 4 * bound, worst


def test_oracle_matches_its_fixture():
    """The oracle reproduces tests/golden/oracle_fixture_p3.txt (written by the committed
    tests/golden/make_oracle_fixture.py, which calls the oracle only): any later change to
    the oracle's arithmetic shows up here."""
    sys.path.insert(0, os.path.dirname(_golden("x")))
    import make_oracle_fixture as mk
    ref = mk.read(_golden("oracle_fixture_p3.txt"))
    got = mk.compute()
    assert set(ref) == set(got)
    for name in ref:
        np.testing.assert_allclose(got[name], ref[name], rtol=0, atol=1e-13, err_msg=name)


def test_chunk_backward_partials_sum_to_the_whole_backward():
    """The ring's backward contributions over every (query chunk, earlier-or-same key
    chunk) pair, with the whole sequence's lse and delta, sum to backward_twopart on the
    whole sequence (a chunk split the plain definition does not know about)."""
    rng = np.random.default_rng(77)
    P, L, H, Hkv, D, theta = 3, 11, 4, 2, 8, 1e4
    q, k, v, do = (rng.standard_normal(s) for s in ((P, L, H, D), (P, L, Hkv, D), (P, L, Hkv, D), (P, L, H, D)))
    O, lse = orc.forward_twopart(q, k, v, theta)
    dq, dk, dv = orc.backward_twopart(q, k, v, do, lse, theta)
    delta = np.einsum("plhd,plhd->phl", do, O)
    cuts = [(0, 3), (3, 4), (7, 4)]
    gq, gk, gv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for a, n in cuts:
        for b, m in cuts:
            if b > a:
                continue
            own = a == b
            r = orc.chunk_backward_partial(q[:, a:a + n], k[0, b:b + m], v[0, b:b + m], do[:, a:a + n],
                                           lse[:, :, a:a + n], delta[:, :, a:a + n], theta, a, b,
                                           branch_k=k[:, a:a + n] if own else None,
                                           branch_v=v[:, a:a + n] if own else None)
            gq[:, a:a + n] += r[0]
            gk[0, b:b + m] += r[1]
            gv[0, b:b + m] += r[2]
            if own:
                gk[1:, a:a + n] += r[3][1:]
                gv[1:, a:a + n] += r[4][1:]
    np.testing.assert_allclose(gq, dq, atol=1e-11)
    np.testing.assert_allclose(gk, dk, atol=1e-11)
    np.testing.assert_allclose(gv, dv, atol=1e-11)
