"""Pins of the fp64 block-draft oracle (DFlash/DSpark anchor + mask-token blocks), CPU
only: each checks it against something other than itself."""

import numpy as np
import pytest
import torch

from oracle import block_draft_oracle as bd

RNG = np.random.default_rng(4321)


def rnd(*shape):
    return RNG.standard_normal(shape)


def case(L=13, nb=3, Bs=4, H=4, Hkv=2, D=8, anchors=None):
    anchors = list(RNG.integers(0, L, nb)) if anchors is None else anchors
    return dict(k_ctx=rnd(L, Hkv, D), v_ctx=rnd(L, Hkv, D), anchors=anchors, qb=rnd(len(anchors), Bs, H, D),
                kb=rnd(len(anchors), Bs, Hkv, D), vb=rnd(len(anchors), Bs, Hkv, D))


def torch_rope(x, pos, theta):
    """Independent RoPE: pair (d, d + D/2) as a complex number times exp(i pos theta^(-2d/D))."""
    D = x.shape[-1]
    freq = torch.tensor([theta ** (-2.0 * d / D) for d in range(D // 2)], dtype=torch.float64)
    ang = torch.tensor(pos, dtype=torch.float64)[:, None] * freq[None, :]
    z = torch.complex(x[..., : D // 2], x[..., D // 2:]) * torch.polar(torch.ones_like(ang), ang)[:, None, :]
    return torch.cat([z.real, z.imag], dim=-1)


@pytest.mark.parametrize("shape", [dict(), dict(L=1, nb=1, Bs=1, H=2, Hkv=1, D=4), dict(L=20, nb=5, Bs=1),
                                   dict(L=9, nb=2, Bs=7, H=3, Hkv=1, D=16)])
def test_twopart_equals_bruteforce(shape):
    c = case(**shape)
    O1, l1 = bd.forward_bruteforce(theta=1e4, **c)
    O2, l2 = bd.forward_twopart(theta=1e4, **c)
    np.testing.assert_allclose(O2, O1, atol=1e-13)
    np.testing.assert_allclose(l2, l1, atol=1e-13)
    do = rnd(*O1.shape)
    g1 = bd.backward_bruteforce(theta=1e4, do=do, **c)
    g2 = bd.backward_twopart(theta=1e4, do=do, O=O2, lse=l2, **c)
    for a, b in zip(g2, g1):
        np.testing.assert_allclose(a, b, atol=1e-12)


@pytest.mark.parametrize("shape", [dict(), dict(L=9, nb=2, Bs=7, H=3, Hkv=1, D=16)])
def test_bf16_rounded_rotation_forms_agree(shape):
    """rope_round="bf16": the brute-force and two-part forms round the same rotated
    arrays, so they still agree, forward and backward."""
    c = case(**shape)
    O1, l1 = bd.forward_bruteforce(theta=1e4, rope_round="bf16", **c)
    O2, l2 = bd.forward_twopart(theta=1e4, rope_round="bf16", **c)
    np.testing.assert_allclose(O2, O1, atol=1e-13)
    np.testing.assert_allclose(l2, l1, atol=1e-13)
    do = rnd(*O1.shape)
    g1 = bd.backward_bruteforce(theta=1e4, do=do, rope_round="bf16", **c)
    g2 = bd.backward_twopart(theta=1e4, do=do, O=O2, lse=l2, rope_round="bf16", **c)
    for a, b in zip(g2, g1):
        np.testing.assert_allclose(a, b, atol=1e-12)


def _bf16_ste(x):
    """torch's own bf16 cast in the forward, identity in the backward."""
    return x + (x.to(torch.bfloat16).double() - x).detach()


@pytest.mark.parametrize("rope_round", [None, "bf16"])
def test_equals_masked_sdpa(rope_round):
    """The block pattern is one masked softmax: torch SDPA (fp64) over the trunk keys and
    the block keys, rotated independently, with the visibility mask written out here,
    outputs and autograd gradients.  With rope_round="bf16" the rotated tensors go
    through torch's bf16 cast (the gradient passing through unchanged), an independent
    restatement of the oracle's rounding step."""
    L, Bs, H, Hkv, D, theta = 10, 3, 4, 2, 8, 1e4
    anchors = [0, 6, 9]
    c = case(L=L, Bs=Bs, H=H, Hkv=Hkv, D=D, anchors=anchors)
    nb = len(anchors)
    O, lse = bd.forward_bruteforce(theta=theta, rope_round=rope_round, **c)
    do = rnd(*O.shape)
    grads = bd.backward_bruteforce(theta=theta, do=do, rope_round=rope_round, **c)
    rnd_ = _bf16_ste if rope_round == "bf16" else (lambda x: x)

    t = {n: torch.tensor(c[n], requires_grad=True) for n in ("k_ctx", "v_ctx", "qb", "kb", "vb")}
    pos_b = [a + j for a in anchors for j in range(Bs)]
    q = rnd_(torch_rope(t["qb"].reshape(nb * Bs, H, D), pos_b, theta))
    k = torch.cat([rnd_(torch_rope(t["k_ctx"], list(range(L)), theta)),
                   rnd_(torch_rope(t["kb"].reshape(nb * Bs, Hkv, D), pos_b, theta))])
    v = torch.cat([t["v_ctx"], t["vb"].reshape(nb * Bs, Hkv, D)])
    mask = torch.zeros(nb * Bs, L + nb * Bs, dtype=torch.bool)
    for b, a in enumerate(anchors):
        for j in range(Bs):
            mask[b * Bs + j, : a + 1] = True                        # trunk up to the anchor
            mask[b * Bs + j, L + b * Bs: L + (b + 1) * Bs] = True   # the whole block
    g = H // Hkv
    out = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(0, 1)[None], k.transpose(0, 1).repeat_interleave(g, 0)[None],
        v.transpose(0, 1).repeat_interleave(g, 0)[None], attn_mask=mask)[0].transpose(0, 1)
    np.testing.assert_allclose(O.reshape(nb * Bs, H, D), out.detach().numpy(), atol=1e-12)
    (out * torch.tensor(do.reshape(nb * Bs, H, D))).sum().backward()
    for got, name in zip(grads, ("qb", "k_ctx", "v_ctx", "kb", "vb")):
        np.testing.assert_allclose(got, t[name].grad.numpy(), atol=1e-11, err_msg=name)


def test_trunk_truncated_at_the_anchor():
    """Trunk keys after the anchor do not reach the block; the anchor's own trunk key does."""
    c = case(L=12, anchors=[4], Bs=3)
    O, _ = bd.forward_twopart(theta=1e4, **c)
    later = dict(c, k_ctx=c["k_ctx"].copy(), v_ctx=c["v_ctx"].copy())
    later["k_ctx"][5:] += 3.0
    later["v_ctx"][5:] -= 2.0
    np.testing.assert_array_equal(bd.forward_twopart(theta=1e4, **later)[0], O)
    at = dict(c, v_ctx=c["v_ctx"].copy())
    at["v_ctx"][4] += 1.0
    assert np.max(np.abs(bd.forward_twopart(theta=1e4, **at)[0] - O)) > 1e-6


def test_block_is_bidirectional_and_isolated():
    """The anchor's query sees the last mask token of its block; no block sees another."""
    c = case(L=8, anchors=[2, 5], Bs=4)
    O, _ = bd.forward_twopart(theta=1e4, **c)
    last = dict(c, vb=c["vb"].copy())
    last["vb"][0, 3] += 1.0
    O2, _ = bd.forward_twopart(theta=1e4, **last)
    assert np.max(np.abs(O2[0, 0] - O[0, 0])) > 1e-6     # anchor query of block 0 moved
    np.testing.assert_array_equal(O2[1], O[1])            # block 1 untouched


def test_uniform_scores_closed_form():
    """q = 0: every visible key scores 0, so O is the mean of the visible values and lse
    the log of their count (a + 1 trunk keys + Bs block keys)."""
    c = case(L=9, anchors=[0, 3, 8], Bs=2, H=2, Hkv=1)
    c["qb"] = np.zeros_like(c["qb"])
    O, lse = bd.forward_twopart(theta=1e4, **c)
    for b, a in enumerate(c["anchors"]):
        vis = np.concatenate([c["v_ctx"][: a + 1, 0], c["vb"][b, :, 0]])
        for j in range(2):
            for h in range(2):
                np.testing.assert_allclose(O[b, j, h], vis.mean(axis=0), atol=1e-14)
                assert abs(lse[b, h, j] - np.log(a + 1 + 2)) < 1e-14


def test_position_shift_invariance():
    """RoPE scores depend on position differences only: shifting every position by a
    constant leaves outputs and gradients unchanged."""
    c = case()
    O0, l0 = bd.forward_twopart(theta=1e4, **c)
    O1, l1 = bd.forward_twopart(theta=1e4, pos_offset=37, **c)
    np.testing.assert_allclose(O1, O0, atol=1e-12)
    np.testing.assert_allclose(l1, l0, atol=1e-12)
    do = rnd(*O0.shape)
    g0 = bd.backward_twopart(theta=1e4, do=do, O=O0, lse=l0, **c)
    g1 = bd.backward_twopart(theta=1e4, do=do, O=O1, lse=l1, pos_offset=37, **c)
    for a, b in zip(g1, g0):
        np.testing.assert_allclose(a, b, atol=1e-11)


def test_finite_differences():
    """Central differences of sum(O * dO) against the two-part analytic gradients."""
    c = case(L=5, anchors=[1, 4], Bs=2, H=2, Hkv=1, D=4)
    O, lse = bd.forward_twopart(theta=1e4, **c)
    do = rnd(*O.shape)
    grads = bd.backward_twopart(theta=1e4, do=do, O=O, lse=lse, **c)
    eps = 1e-6
    for name, g in zip(("qb", "k_ctx", "v_ctx", "kb", "vb"), grads):
        fd = np.zeros_like(c[name])
        for idx in np.ndindex(c[name].shape):
            plus, minus = dict(c), dict(c)
            plus[name] = c[name].copy()
            minus[name] = c[name].copy()
            plus[name][idx] += eps
            minus[name][idx] -= eps
            fd[idx] = (np.sum(bd.forward_bruteforce(theta=1e4, **plus)[0] * do) -
                       np.sum(bd.forward_bruteforce(theta=1e4, **minus)[0] * do)) / (2 * eps)
        np.testing.assert_allclose(g, fd, atol=2e-8, err_msg=name)


def test_oracle_matches_its_fixture():
    """The oracle reproduces tests/golden/block_draft_fixture.txt (written by the committed
    tests/golden/make_block_draft_fixture.py, which calls the oracle only)."""
    import os
    import sys
    golden = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
    sys.path.insert(0, golden)
    import make_block_draft_fixture as mk
    ref = mk.read(os.path.join(golden, "block_draft_fixture.txt"))
    got = mk.compute()
    assert set(ref) == set(got)
    for name in ref:
        np.testing.assert_allclose(got[name], ref[name], rtol=0, atol=1e-13, err_msg=name)


# ----------------------------------------------------------------------------- sliding-window trunk
@pytest.mark.parametrize("window", [1, 3, 6])
def test_window_equals_masked_sdpa(window):
    """A sliding-window layer is one masked softmax too: torch SDPA (fp64) with the trunk
    part of the mask written out here as a - window < t <= a, outputs and autograd
    gradients against both oracle forms."""
    L, Bs, H, Hkv, D, theta = 11, 3, 4, 2, 8, 1e4
    anchors = [0, 2, 7, 10]
    c = case(L=L, Bs=Bs, H=H, Hkv=Hkv, D=D, anchors=anchors)
    nb = len(anchors)
    O, lse = bd.forward_twopart(theta=theta, window=window, **c)
    Ob, lb = bd.forward_bruteforce(theta=theta, window=window, **c)
    np.testing.assert_allclose(Ob, O, atol=1e-13)
    np.testing.assert_allclose(lb, lse, atol=1e-13)
    do = rnd(*O.shape)
    grads = bd.backward_twopart(theta=theta, do=do, O=O, lse=lse, window=window, **c)
    grads_b = bd.backward_bruteforce(theta=theta, do=do, window=window, **c)
    t = {n: torch.tensor(c[n], requires_grad=True) for n in ("k_ctx", "v_ctx", "qb", "kb", "vb")}
    pos_b = [a + j for a in anchors for j in range(Bs)]
    q = torch_rope(t["qb"].reshape(nb * Bs, H, D), pos_b, theta)
    k = torch.cat([torch_rope(t["k_ctx"], list(range(L)), theta),
                   torch_rope(t["kb"].reshape(nb * Bs, Hkv, D), pos_b, theta)])
    v = torch.cat([t["v_ctx"], t["vb"].reshape(nb * Bs, Hkv, D)])
    mask = torch.zeros(nb * Bs, L + nb * Bs, dtype=torch.bool)
    for b, a in enumerate(anchors):
        for j in range(Bs):
            for tt in range(L):
                mask[b * Bs + j, tt] = a - window < tt <= a
            mask[b * Bs + j, L + b * Bs: L + (b + 1) * Bs] = True
    g = H // Hkv
    out = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(0, 1)[None], k.transpose(0, 1).repeat_interleave(g, 0)[None],
        v.transpose(0, 1).repeat_interleave(g, 0)[None], attn_mask=mask)[0].transpose(0, 1)
    np.testing.assert_allclose(O.reshape(nb * Bs, H, D), out.detach().numpy(), atol=1e-12)
    (out * torch.tensor(do.reshape(nb * Bs, H, D))).sum().backward()
    for got, got_b, name in zip(grads, grads_b, ("qb", "k_ctx", "v_ctx", "kb", "vb")):
        np.testing.assert_allclose(got, t[name].grad.numpy(), atol=1e-11, err_msg=name)
        np.testing.assert_allclose(got_b, t[name].grad.numpy(), atol=1e-11, err_msg=name)


def test_window_covering_the_trunk_is_the_full_layer():
    """A window of at least anchor + 1 keys changes nothing (bit for bit), and so does 0."""
    c = case(L=9, anchors=[0, 4, 8], Bs=2)
    O, lse = bd.forward_twopart(theta=1e4, **c)
    for w in (0, 9, 50):
        O2, l2 = bd.forward_twopart(theta=1e4, window=w, **c)
        np.testing.assert_array_equal(O2, O)
        np.testing.assert_array_equal(l2, lse)


def test_window_uniform_scores_closed_form():
    """q = 0: O is the mean of the min(window, a + 1) trunk values in the window and the
    Bs block values, lse the log of their count."""
    c = case(L=12, anchors=[1, 5, 11], Bs=2, H=2, Hkv=1)
    c["qb"] = np.zeros_like(c["qb"])
    w = 4
    O, lse = bd.forward_twopart(theta=1e4, window=w, **c)
    for b, a in enumerate(c["anchors"]):
        t0 = max(0, a - w + 1)
        vis = np.concatenate([c["v_ctx"][t0: a + 1, 0], c["vb"][b, :, 0]])
        for j in range(2):
            for h in range(2):
                np.testing.assert_allclose(O[b, j, h], vis.mean(axis=0), atol=1e-14)
                assert abs(lse[b, h, j] - np.log(a + 1 - t0 + 2)) < 1e-14


def test_window_one_sees_the_anchor_key_only():
    """window = 1: the trunk part is the anchor's key alone, so its lse is that one score
    and keys before the anchor do not matter."""
    c = case(L=10, anchors=[3, 9], Bs=2, H=2, Hkv=1, D=8)
    O, lse, parts = bd.forward_twopart(theta=1e4, window=1, return_parts=True, **c)
    kt, qr, _ = bd._rotate(c["k_ctx"], c["anchors"], c["qb"], c["kb"], 1e4)
    sc = 1.0 / np.sqrt(8)
    for b, h, lt, _ in parts:
        a = c["anchors"][b]
        np.testing.assert_allclose(lt, sc * qr[b, :, h] @ kt[a, h // 2], atol=1e-13)
    before = dict(c, k_ctx=c["k_ctx"].copy(), v_ctx=c["v_ctx"].copy())
    before["k_ctx"][:3] += 5.0
    before["v_ctx"][4:9] -= 2.0
    np.testing.assert_array_equal(bd.forward_twopart(theta=1e4, window=1, **before)[0], O)
