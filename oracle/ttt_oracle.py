"""fp64 CPU oracle for multi-pass TTT trunk+branch attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this module.  The
library (``attention_pass_rope_b200``) never imports it and shares no code with
it; the only module both sides use is ``ttt_inputs`` (seeded random draws).

What is computed (sources, by page and section):

* "DFlash/DSpark and EAGLE-3 TTT draft co-training for speculative decoding
  (Megatron backend)" (NeMo-RL issue 3698), section "What I'm working on",
  item 1: P sequential draft passes; a two-part trunk+branch attention whose two
  partial softmaxes are merged exactly through their log-sum-exps; each pass
  uses RoPE position offsets aligned with inference.  Item 4: the same
  attention on the packed varlen (THD) layout, pass-1 trunk K/V as the part
  that is shared.
* "bounded multi-pass EAGLE-3 TTT provider" (NeMo-RL PR 3725), Summary: no
  dense pass logits, no sequence-square masks; self-review: the multi-pass
  "staircase" visibility and the RoPE relative shift, checked against an
  independent rotate-half oracle in fp64.
* The benchmark spec fixes the offsets: at pass p (1-based) the query at
  position i is rotated to position i+p-1; it sees the pass-1 trunk keys
  0..i (causal) and, on the staircase diagonal, the branch keys of passes
  2..p at the same position i.

Readings where the pages are silent:

* RoPE is rotate-half (dimension d pairs with d + D/2) with inverse frequency
  theta**(-2k/D), k < D/2, over the whole head dimension.
* The key of pass j at position i is rotated to the same position as the
  query of pass j, i+j-1 (so trunk key t sits at t).  Scores therefore depend
  on (i+p-1) - t for the trunk and on p - j for the branch.
* The softmax scale is 1/sqrt(D) unless given; lse is the natural log of the
  sum of exp(scaled score).
* GQA: query head h reads KV head h // (H // Hkv).
* THD: positions restart at 0 at every sequence start; nothing crosses
  sequences.
* ``rope_round="bf16"`` rounds the rotated q/k to bf16 (round to nearest
  even) before the attention, the library's defined semantics (bf16 operands
  into the tensor cores).  ``rope_round=None`` keeps them exact.  Gradients
  treat that rounding as the identity.

Two forms that share nothing but the RoPE helper and the input arrays:

* :func:`forward_bruteforce` / :func:`backward_bruteforce`: all P*L keys of a
  sequence concatenated, an explicit boolean staircase mask, one dense
  softmax.  Tiny inputs only.
* :func:`forward_twopart` / :func:`backward_twopart`: the method itself: a
  causal trunk softmax (lse_t, O_t), a branch softmax over the <= P-1
  diagonal keys (lse_b, O_b), merged by lse = logaddexp(lse_t, lse_b).

Array conventions (one sequence): q [P, L, H, D], k and v [P, L, Hkv, D];
index 0 along P is the trunk pass.  Outputs: O [P, L, H, D], lse [P, H, L].
"""

from __future__ import annotations

import math

import numpy as np

# --------------------------------------------------------------------------
# bf16 rounding (round to nearest, ties to even) written with integer ops
# --------------------------------------------------------------------------


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round to the nearest bf16 value (ties to even); returns fp64.

    fp64 -> fp32 (numpy, round to nearest even) -> keep the top 16 bits of the
    fp32 pattern after adding 0x7fff plus the lowest kept bit (the usual
    round-half-to-even on the dropped 16 bits).  Finite inputs only.
    """
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    bits = (bits + 0x7FFF + lsb) & 0xFFFF0000
    return bits.astype(np.uint32).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# RoPE (rotate-half), positions per pass
# --------------------------------------------------------------------------


def rope_inv_freq(D: int, theta: float) -> np.ndarray:
    k = np.arange(D // 2, dtype=np.float64)
    return float(theta) ** (-2.0 * k / D)


def rope_rotate(x: np.ndarray, pos: np.ndarray, theta: float, inverse: bool = False) -> np.ndarray:
    """Rotate-half RoPE of ``x[..., L, nh, D]`` at integer positions ``pos[L]``.

    Pair (d, d + D/2) is rotated by the angle pos * inv_freq[d]:
    (x1, x2) -> (x1 cos - x2 sin, x2 cos + x1 sin).  ``inverse`` applies the
    transpose (rotation by the negative angle), which is also the adjoint used
    to carry gradients back to the pre-RoPE inputs.
    """
    D = x.shape[-1]
    ang = np.outer(np.asarray(pos, dtype=np.float64), rope_inv_freq(D, theta))  # [L, D/2]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    if inverse:
        s = -s
    x1 = x[..., : D // 2]
    x2 = x[..., D // 2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def pass_positions(L: int, p0: int, pos_offset: int = 0) -> np.ndarray:
    """Positions of pass ``p0`` (0-based; pass p0+1 in 1-based terms): i + p0."""
    return np.arange(L, dtype=np.int64) + p0 + pos_offset


def rotate_inputs(q, k, theta, rope_round="bf16", pos_offset=0):
    """Rotated q~, k~ of one sequence (every pass at its own offset)."""
    P, L = q.shape[0], q.shape[1]
    qr = np.empty_like(q, dtype=np.float64)
    kr = np.empty_like(k, dtype=np.float64)
    for p0 in range(P):
        pos = pass_positions(L, p0, pos_offset)
        qr[p0] = rope_rotate(q[p0].astype(np.float64), pos, theta)
        kr[p0] = rope_rotate(k[p0].astype(np.float64), pos, theta)
    if rope_round == "bf16":
        qr = bf16_round(qr)
        kr = bf16_round(kr)
    elif rope_round is not None:
        raise ValueError(rope_round)
    return qr, kr


def unrotate_grads(dqr, dkr, theta, pos_offset=0):
    P, L = dqr.shape[0], dqr.shape[1]
    dq = np.empty_like(dqr)
    dk = np.empty_like(dkr)
    for p0 in range(P):
        pos = pass_positions(L, p0, pos_offset)
        dq[p0] = rope_rotate(dqr[p0], pos, theta, inverse=True)
        dk[p0] = rope_rotate(dkr[p0], pos, theta, inverse=True)
    return dq, dk


def _scale(D, scale):
    return 1.0 / math.sqrt(D) if scale is None else float(scale)


# --------------------------------------------------------------------------
# (i) brute force: concatenated keys + explicit staircase mask
# --------------------------------------------------------------------------


def staircase_mask(P: int, L: int) -> np.ndarray:
    """Boolean [(P*L), (P*L)] visibility, rows (p, i), columns (j, t), 0-based passes.

    Query (p, i) sees trunk key (0, t) for t <= i, and branch key (j, t) iff
    1 <= j <= p and t == i.
    """
    p = np.repeat(np.arange(P), L)[:, None]
    i = np.tile(np.arange(L), P)[:, None]
    j = np.repeat(np.arange(P), L)[None, :]
    t = np.tile(np.arange(L), P)[None, :]
    trunk = (j == 0) & (t <= i)
    branch = (j >= 1) & (j <= p) & (t == i)
    return trunk | branch


def forward_bruteforce(q, k, v, theta, scale=None, rope_round="bf16", pos_offset=0):
    P, L, H, D = q.shape
    Hkv = k.shape[2]
    g = H // Hkv
    sc = _scale(D, scale)
    qr, kr = rotate_inputs(q, k, theta, rope_round, pos_offset)
    vv = v.astype(np.float64)
    mask = staircase_mask(P, L)
    O = np.zeros((P, L, H, D))
    lse = np.zeros((P, H, L))
    for h in range(H):
        kv = h // g
        Qc = qr[:, :, h, :].reshape(P * L, D)
        Kc = kr[:, :, kv, :].reshape(P * L, D)
        Vc = vv[:, :, kv, :].reshape(P * L, D)
        S = np.where(mask, sc * (Qc @ Kc.T), -np.inf)
        m = S.max(axis=1, keepdims=True)
        E = np.exp(S - m)
        Z = E.sum(axis=1, keepdims=True)
        A = E / Z
        O[:, :, h, :] = (A @ Vc).reshape(P, L, D)
        lse[:, h, :] = (m[:, 0] + np.log(Z[:, 0])).reshape(P, L)
    return O, lse


def backward_bruteforce(q, k, v, do, theta, scale=None, rope_round="bf16", pos_offset=0):
    """Analytic softmax-attention gradient on the concatenated form, w.r.t. the
    pre-RoPE q, k and v."""
    P, L, H, D = q.shape
    Hkv = k.shape[2]
    g = H // Hkv
    sc = _scale(D, scale)
    qr, kr = rotate_inputs(q, k, theta, rope_round, pos_offset)
    vv = v.astype(np.float64)
    dd = do.astype(np.float64)
    mask = staircase_mask(P, L)
    dqr = np.zeros((P, L, H, D))
    dkr = np.zeros((P, L, Hkv, D))
    dv = np.zeros((P, L, Hkv, D))
    for h in range(H):
        kv = h // g
        Qc = qr[:, :, h, :].reshape(P * L, D)
        Kc = kr[:, :, kv, :].reshape(P * L, D)
        Vc = vv[:, :, kv, :].reshape(P * L, D)
        dOc = dd[:, :, h, :].reshape(P * L, D)
        S = np.where(mask, sc * (Qc @ Kc.T), -np.inf)
        m = S.max(axis=1, keepdims=True)
        E = np.exp(S - m)
        A = E / E.sum(axis=1, keepdims=True)
        dA = dOc @ Vc.T
        delta = (A * dA).sum(axis=1, keepdims=True)
        dS = A * (dA - delta)
        dqr[:, :, h, :] = (sc * (dS @ Kc)).reshape(P, L, D)
        dkr[:, :, kv, :] += (sc * (dS.T @ Qc)).reshape(P, L, D)
        dv[:, :, kv, :] += (A.T @ dOc).reshape(P, L, D)
    dq, dk = unrotate_grads(dqr, dkr, theta, pos_offset)
    return dq, dk, dv


# --------------------------------------------------------------------------
# (ii) the method: trunk softmax + branch softmax, exact joint-LSE merge
# --------------------------------------------------------------------------


def _logsumexp_rows(S):
    m = S.max(axis=-1, keepdims=True)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    with np.errstate(divide="ignore"):
        return (m_safe + np.log(np.exp(S - m_safe).sum(axis=-1, keepdims=True)))[..., 0]


def _trunk_block(qr_blk, kr1, i0, sc):
    """Scores of query rows i0..i0+nb-1 against trunk keys 0..L-1, causal."""
    nb = qr_blk.shape[0]
    L = kr1.shape[0]
    S = sc * (qr_blk @ kr1.T)
    rows = np.arange(i0, i0 + nb)[:, None]
    cols = np.arange(L)[None, :]
    return np.where(cols <= rows, S, -np.inf)


def forward_twopart(q, k, v, theta, scale=None, rope_round="bf16", pos_offset=0,
                    heads=None, block=1024, return_parts=False):
    """Trunk + branch + merge.  ``heads`` restricts the query heads computed
    (others are left NaN); ``return_parts`` also returns (O_t, lse_t, O_b, lse_b)."""
    P, L, H, D = q.shape
    Hkv = k.shape[2]
    g = H // Hkv
    sc = _scale(D, scale)
    qr, kr = rotate_inputs(q, k, theta, rope_round, pos_offset)
    vv = v.astype(np.float64)
    heads = range(H) if heads is None else heads
    O = np.full((P, L, H, D), np.nan)
    lse = np.full((P, H, L), np.nan)
    parts = {n: np.full(s, np.nan) for n, s in
             (("O_t", (P, L, H, D)), ("lse_t", (P, H, L)), ("O_b", (P, L, H, D)), ("lse_b", (P, H, L)))}
    for h in heads:
        kv = h // g
        kr1 = kr[0, :, kv, :]
        v1 = vv[0, :, kv, :]
        for p0 in range(P):
            # trunk: causal softmax over pass-1 keys 0..i
            O_t = np.empty((L, D))
            lse_t = np.empty(L)
            for i0 in range(0, L, block):
                S = _trunk_block(qr[p0, i0:i0 + block, h, :], kr1[: min(L, i0 + block)], i0, sc)
                ls = _logsumexp_rows(S)
                O_t[i0:i0 + block] = np.exp(S - ls[:, None]) @ v1[: min(L, i0 + block)]
                lse_t[i0:i0 + block] = ls
            # branch: passes 1..p0 (0-based) at the same position
            if p0 == 0:
                lse_b = np.full(L, -np.inf)
                O_b = np.zeros((L, D))
            else:
                kb = kr[1:p0 + 1, :, kv, :]                      # [p0, L, D]
                vb = vv[1:p0 + 1, :, kv, :]
                s_b = sc * np.einsum("ld,jld->lj", qr[p0, :, h, :], kb)
                lse_b = _logsumexp_rows(s_b)
                w = np.exp(s_b - lse_b[:, None])                 # [L, p0]
                O_b = np.einsum("lj,jld->ld", w, vb)
            # exact merge of the two partial softmaxes
            lse_m = np.logaddexp(lse_t, lse_b)
            O[p0, :, h, :] = np.exp(lse_t - lse_m)[:, None] * O_t + np.exp(lse_b - lse_m)[:, None] * O_b
            lse[p0, h, :] = lse_m
            parts["O_t"][p0, :, h, :] = O_t
            parts["lse_t"][p0, h, :] = lse_t
            parts["O_b"][p0, :, h, :] = O_b
            parts["lse_b"][p0, h, :] = lse_b
    if return_parts:
        return O, lse, parts
    return O, lse


def backward_twopart(q, k, v, do, lse, theta, scale=None, rope_round="bf16", pos_offset=0,
                     kv_heads=None, block=1024):
    """Gradient of the merged attention w.r.t. pre-RoPE q, k, v, recomputing the
    probabilities from the merged lse.

    ``kv_heads`` restricts the work to the query heads of those KV heads: dq is
    then exact for those query heads, dk/dv exact for those KV heads (others NaN).
    """
    P, L, H, D = q.shape
    Hkv = k.shape[2]
    g = H // Hkv
    sc = _scale(D, scale)
    qr, kr = rotate_inputs(q, k, theta, rope_round, pos_offset)
    vv = v.astype(np.float64)
    dd = do.astype(np.float64)
    kv_heads = range(Hkv) if kv_heads is None else kv_heads
    dqr = np.full((P, L, H, D), np.nan)
    dkr = np.full((P, L, Hkv, D), np.nan)
    dv = np.full((P, L, Hkv, D), np.nan)
    for kv in kv_heads:
        dkr[:, :, kv, :] = 0.0
        dv[:, :, kv, :] = 0.0
        kr1 = kr[0, :, kv, :]
        v1 = vv[0, :, kv, :]
        for h in range(kv * g, (kv + 1) * g):
            for p0 in range(P):
                ls = lse[p0, h, :]
                dO = dd[p0, :, h, :]
                qh = qr[p0, :, h, :]
                # branch part (keys of passes 1..p0 at the same position)
                if p0 > 0:
                    kb = kr[1:p0 + 1, :, kv, :]
                    vb = vv[1:p0 + 1, :, kv, :]
                    Pb = np.exp(sc * np.einsum("ld,jld->lj", qh, kb) - ls[:, None])   # [L, p0]
                    dPb = np.einsum("ld,jld->lj", dO, vb)
                else:
                    Pb = np.zeros((L, 0))
                    dPb = np.zeros((L, 0))
                delta = (Pb * dPb).sum(axis=1)      # branch share of each row's delta
                dq_rows = np.zeros((L, D))
                for i0 in range(0, L, block):
                    n = min(L, i0 + block)
                    rows = slice(i0, i0 + block)
                    Pt = np.exp(_trunk_block(qh[rows], kr1[:n], i0, sc) - ls[rows, None])
                    dPt = dO[rows] @ v1[:n].T
                    # delta of a row = sum over all its visible keys of P * dP
                    delta[rows] += (Pt * dPt).sum(axis=1)
                    dSt = Pt * (dPt - delta[rows, None])
                    dq_rows[rows] += sc * (dSt @ kr1[:n])
                    dkr[0, :n, kv, :] += sc * (dSt.T @ qh[rows])
                    dv[0, :n, kv, :] += Pt.T @ dO[rows]
                if p0 > 0:
                    dSb = Pb * (dPb - delta[:, None])                                   # [L, p0]
                    dq_rows += sc * np.einsum("lj,jld->ld", dSb, kb)
                    dkr[1:p0 + 1, :, kv, :] += sc * np.einsum("lj,ld->jld", dSb, qh)
                    dv[1:p0 + 1, :, kv, :] += np.einsum("lj,ld->jld", Pb, dO)
                dqr[p0, :, h, :] = dq_rows
    dq, dk = unrotate_grads(dqr, dkr, theta, pos_offset)
    return dq, dk, dv


# --------------------------------------------------------------------------
# packed batches: dense [B, S] or THD (cu_seqlens), public lse layouts
# --------------------------------------------------------------------------


def _seq_slices(cu_seqlens):
    return [(int(cu_seqlens[n]), int(cu_seqlens[n + 1])) for n in range(len(cu_seqlens) - 1)]


def lse_to_public(lse_seq, cu_seqlens, dense):
    """Per-sequence lse [P, H, L] list -> dense [P, B, H, S] or THD [P, H, T]."""
    if dense:
        return np.stack(lse_seq, axis=1)
    return np.concatenate(lse_seq, axis=2)


def lse_from_public(lse, cu_seqlens, dense):
    if dense:
        return [lse[:, b] for b in range(lse.shape[1])]
    return [lse[:, :, a:b] for a, b in _seq_slices(cu_seqlens)]


def forward_packed(q, k, v, cu_seqlens, theta, dense, scale=None, rope_round="bf16", heads=None,
                   seqs=None):
    """q [P, T, H, D], k, v [P, T, Hkv, D] -> O [P, T, H, D], lse (public layout).

    ``seqs`` restricts the sequences computed (others NaN)."""
    P, T, H, D = q.shape
    O = np.full((P, T, H, D), np.nan)
    lse_seq = []
    for n, (a, b) in enumerate(_seq_slices(cu_seqlens)):
        if seqs is not None and n not in seqs:
            lse_seq.append(np.full((P, H, b - a), np.nan))
            continue
        O_s, lse_s = forward_twopart(q[:, a:b], k[:, a:b], v[:, a:b], theta, scale, rope_round,
                                     heads=heads)
        O[:, a:b] = O_s
        lse_seq.append(lse_s)
    return O, lse_to_public(lse_seq, cu_seqlens, dense)


def backward_packed(q, k, v, do, lse, cu_seqlens, theta, dense, scale=None, rope_round="bf16",
                    kv_heads=None, seqs=None):
    P, T, H, D = q.shape
    Hkv = k.shape[2]
    dq = np.full((P, T, H, D), np.nan)
    dk = np.full((P, T, Hkv, D), np.nan)
    dv = np.full((P, T, Hkv, D), np.nan)
    lse_seq = lse_from_public(lse, cu_seqlens, dense)
    for n, (a, b) in enumerate(_seq_slices(cu_seqlens)):
        if seqs is not None and n not in seqs:
            continue
        g = backward_twopart(q[:, a:b], k[:, a:b], v[:, a:b], do[:, a:b], lse_seq[n], theta, scale,
                             rope_round, kv_heads=kv_heads)
        dq[:, a:b], dk[:, a:b], dv[:, a:b] = g
    return dq, dk, dv


# --------------------------------------------------------------------------
# single rows straight from the definition (for samples of full-size workloads)
# --------------------------------------------------------------------------


def _rot_rows(x_rows, positions, theta, rope_round):
    """Rotate rows x_rows[n, D] at positions[n] (one position per row)."""
    out = np.empty_like(x_rows, dtype=np.float64)
    for n, m in enumerate(positions):
        out[n] = rope_rotate(x_rows[n][None, None, :].astype(np.float64), [int(m)], theta)[0, 0]
    if rope_round == "bf16":
        out = bf16_round(out)
    return out


def rotate_trunk_keys(k, kv, theta, rope_round="bf16"):
    """Rotated trunk keys k~_1[0..L-1] of KV head kv (key t at position t)."""
    L = k.shape[1]
    return _rot_rows(k[0, :, kv], np.arange(L), theta, rope_round)


def _visible(q, k, v, theta, sc, rope_round, p0, i, h, g, kt=None):
    """Rotated query row, visible keys and values of query (pass p0, position i, head h).
    ``kt``: rotated trunk keys of the KV head (rotate_trunk_keys), computed if absent."""
    kv = h // g
    qr = _rot_rows(q[p0, i, h][None, :], [i + p0], theta, rope_round)[0]
    if kt is None:
        kt = _rot_rows(k[0, : i + 1, kv], np.arange(i + 1), theta, rope_round)   # trunk keys 0..i
    keys = [kt[: i + 1]]
    vals = [v[0, : i + 1, kv].astype(np.float64)]
    if p0 > 0:                                                                     # branch keys j = 1..p0
        kb = np.stack([k[j, i, kv] for j in range(1, p0 + 1)])
        keys.append(_rot_rows(kb, [i + j for j in range(1, p0 + 1)], theta, rope_round))
        vals.append(np.stack([v[j, i, kv] for j in range(1, p0 + 1)]).astype(np.float64))
    return qr, np.concatenate(keys), np.concatenate(vals)


def row_forward(q, k, v, theta, p0, i, h, scale=None, rope_round="bf16", kt=None):
    """O[p0, i, h, :] and lse[p0, h, i] of one sequence by the plain definition."""
    H, D = q.shape[2], q.shape[3]
    g = H // k.shape[2]
    sc = _scale(D, scale)
    qr, K, V = _visible(q, k, v, theta, sc, rope_round, p0, i, h, g, kt)
    s = sc * (K @ qr)
    m = s.max()
    e = np.exp(s - m)
    return (e / e.sum()) @ V, m + np.log(e.sum())


def _row_grads(q, k, v, do, theta, sc, rope_round, p0, i, h, g, kt=None):
    """Softmax and its gradient pieces for one query row: (qr, K, V, P, dS)."""
    qr, K, V = _visible(q, k, v, theta, sc, rope_round, p0, i, h, g, kt)
    s = sc * (K @ qr)
    P = np.exp(s - s.max())
    P /= P.sum()
    dP = V @ do[p0, i, h].astype(np.float64)
    dS = P * (dP - np.dot(P, dP))
    return qr, K, V, P, dS


def row_dq(q, k, v, do, theta, p0, i, h, scale=None, rope_round="bf16", kt=None):
    """dQ[p0, i, h, :] (w.r.t. the pre-RoPE query) of one sequence."""
    H, D = q.shape[2], q.shape[3]
    g = H // k.shape[2]
    sc = _scale(D, scale)
    _, K, _, _, dS = _row_grads(q, k, v, do, theta, sc, rope_round, p0, i, h, g, kt)
    dqr = sc * (dS @ K)
    return rope_rotate(dqr[None, None, :], [i + p0], theta, inverse=True)[0, 0]


def row_dkv(q, k, v, do, theta, j0, t, kv, scale=None, rope_round="bf16"):
    """dK[j0, t, kv, :] (pre-RoPE) and dV[j0, t, kv, :] of one sequence: the sum over
    every query row that sees key (pass j0, position t) of KV head kv."""
    P_, L, H, D = q.shape
    g = H // k.shape[2]
    sc = _scale(D, scale)
    dkr = np.zeros(D)
    dv = np.zeros(D)
    kt = rotate_trunk_keys(k, kv, theta, rope_round)
    for h in range(kv * g, (kv + 1) * g):
        if j0 == 0:
            rows = [(p0, i) for p0 in range(P_) for i in range(t, L)]   # trunk key t: every query i >= t
            col = lambda p0, i: t                                        # index among the visible keys
        else:
            rows = [(p0, t) for p0 in range(j0, P_)]                      # branch key: queries at position t
            col = lambda p0, i: (i + 1) + (j0 - 1)
        for p0, i in rows:
            qr, K, V, Pr, dS = _row_grads(q, k, v, do, theta, sc, rope_round, p0, i, h, g, kt)
            c = col(p0, i)
            dkr += sc * dS[c] * qr
            dv += Pr[c] * do[p0, i, h].astype(np.float64)
    dk = rope_rotate(dkr[None, None, :], [t + j0], theta, inverse=True)[0, 0]
    return dk, dv


def tail_trunk_dkv(q, k, v, do, theta, kv, t0, scale=None, rope_round="bf16"):
    """dK[0, t0:, kv, :] (pre-RoPE) and dV[0, t0:, kv, :] of one sequence: the trunk
    keys t >= t0 of KV head kv, summed over every query row that sees them (rows
    i >= t0 of every pass and every query head of the group).

    Plain definition, vectorised over the rows i = t0..L-1 of one (pass, head) at a
    time: each row's softmax runs over all its visible keys (trunk 0..i and the
    branch keys of passes 2..p at position i), dS = P (dP - delta) with delta the sum
    of P dP over those keys, then dk~_1[t] = sigma * sum_rows dS[., t] q~,
    dV_1[t] = sum_rows P[., t] dO, and dK = R(t)^T dk~.  Used on the last keys of
    long sequences, where few rows see them."""
    P_, L, H, D = q.shape
    g = H // k.shape[2]
    sc = _scale(D, scale)
    rows = np.arange(t0, L)
    kt = rope_rotate(k[0, :, kv][:, None, :].astype(np.float64), np.arange(L), theta)[:, 0]
    if rope_round == "bf16":
        kt = bf16_round(kt)
    v1 = v[0, :, kv].astype(np.float64)
    causal = np.arange(L)[None, :] <= rows[:, None]                       # [R, L]
    dkr = np.zeros((L - t0, D))
    dv = np.zeros((L - t0, D))
    for h in range(kv * g, (kv + 1) * g):
        for p0 in range(P_):
            qr = rope_rotate(q[p0, t0:, h][:, None, :].astype(np.float64), rows + p0, theta)[:, 0]
            if rope_round == "bf16":
                qr = bf16_round(qr)
            dO = do[p0, t0:, h].astype(np.float64)
            s_t = np.where(causal, sc * (qr @ kt.T), -np.inf)                  # [R, L]
            dp_t = dO @ v1.T
            if p0 > 0:                                                          # branch keys j = 1..p0
                kb = np.stack([rope_rotate(k[j, t0:, kv][:, None, :].astype(np.float64), rows + j, theta)[:, 0]
                               for j in range(1, p0 + 1)], axis=1)              # [R, p0, D]
                if rope_round == "bf16":
                    kb = bf16_round(kb)
                vb = np.stack([v[j, t0:, kv] for j in range(1, p0 + 1)], axis=1).astype(np.float64)
                s_b = sc * np.einsum("rd,rjd->rj", qr, kb)
                dp_b = np.einsum("rd,rjd->rj", dO, vb)
            else:
                s_b = np.zeros((L - t0, 0))
                dp_b = np.zeros((L - t0, 0))
            s_all = np.concatenate([s_t, s_b], axis=1)
            m = s_all.max(axis=1, keepdims=True)
            e = np.exp(s_all - m)
            Pr = e / e.sum(axis=1, keepdims=True)
            dp_all = np.concatenate([dp_t, dp_b], axis=1)
            delta = (Pr * dp_all).sum(axis=1, keepdims=True)
            dS_t = Pr[:, :L] * (dp_t - delta)
            dkr += sc * (dS_t[:, t0:].T @ qr)
            dv += Pr[:, t0:L].T @ dO
    dk = rope_rotate(dkr[:, None, :], rows, theta, inverse=True)[:, 0]
    return dk, dv


# --------------------------------------------------------------------------
# context-parallel ring: the partial attention of one query chunk over one
# chunk of trunk keys (NeMo-RL issue 3698, "What I'm working on", item 4)
# --------------------------------------------------------------------------


def chunk_partial(qc, kt, vt, theta, q_start, kv_start, branch_k=None, branch_v=None, scale=None,
                  rope_round="bf16"):
    """Partial attention of the query chunk qc [P, Lq, H, D] (pre-RoPE; row i of pass p0
    at global position q_start + i + p0) over the trunk-key chunk kt, vt [Lk, Hkv, D]
    (pass-1 keys at global positions kv_start + t): trunk key t is visible to row i iff
    kv_start + t <= q_start + i.  With branch_k / branch_v ([P, Lq, Hkv, D], the chunk's
    own keys and values of every pass) the branch keys of passes 2..p at the row's own
    position join the partial.  Returns O [P, Lq, H, D] normalised over the visible keys
    and lse [P, H, Lq] (-inf, with O = 0, for a row that sees no key)."""
    P, Lq, H, D = qc.shape
    Lk, Hkv = kt.shape[0], kt.shape[1]
    g = H // Hkv
    sc = _scale(D, scale)
    ktr = rope_rotate(kt.astype(np.float64), np.arange(Lk) + kv_start, theta)
    if branch_k is not None:
        kbr = np.stack([rope_rotate(branch_k[j].astype(np.float64), np.arange(Lq) + q_start + j, theta)
                        for j in range(P)])
    qr = np.stack([rope_rotate(qc[p0].astype(np.float64), np.arange(Lq) + q_start + p0, theta) for p0 in range(P)])
    if rope_round == "bf16":
        ktr, qr = bf16_round(ktr), bf16_round(qr)
        if branch_k is not None:
            kbr = bf16_round(kbr)
    visible = (kv_start + np.arange(Lk))[None, :] <= (q_start + np.arange(Lq))[:, None]   # [Lq, Lk]
    O = np.zeros((P, Lq, H, D))
    lse = np.full((P, H, Lq), -np.inf)
    for h in range(H):
        kv = h // g
        for p0 in range(P):
            s = np.where(visible, sc * (qr[p0, :, h] @ ktr[:, kv].T), -np.inf)              # [Lq, Lk]
            vals = [vt[:, kv].astype(np.float64)]
            if branch_k is not None and p0 > 0:
                sb = sc * np.einsum("ld,jld->lj", qr[p0, :, h], kbr[1:p0 + 1, :, kv])      # [Lq, p0]
                s = np.concatenate([s, sb], axis=1)
            m = s.max(axis=1, keepdims=True)
            has = np.isfinite(m[:, 0])
            e = np.exp(s - np.where(np.isfinite(m), m, 0.0))
            z = e.sum(axis=1)
            w = e / np.where(z > 0, z, 1.0)[:, None]
            out = w[:, :Lk] @ vals[0]
            if branch_k is not None and p0 > 0:
                out += np.einsum("lj,jld->ld", w[:, Lk:], branch_v[1:p0 + 1, :, kv].astype(np.float64))
            O[p0, :, h] = out
            lse[p0, h] = np.where(has, m[:, 0] + np.log(np.where(z > 0, z, 1.0)), -np.inf)
    return O, lse


def chunk_backward_partial(qc, kt, vt, doc, lse_c, delta_c, theta, q_start, kv_start, branch_k=None,
                           branch_v=None, scale=None, rope_round="bf16"):
    """Backward contribution of one (query chunk, trunk-key chunk) pair of the context-
    parallel ring (NeMo-RL issue 3698, "What I'm working on", item 4), given the query
    rows' FINAL lse and delta = rowsum(dO * O) over the whole sequence.

    Plain definition over the pair's visible entries (kv_start + t <= q_start + i):
    P = exp(sigma q~.k~ - lse), dS = P (dO.V - delta), dq~ = sigma dS k~,
    dk~ = sigma dS^T q~ (summed over every pass and query head of the group),
    dV = P^T dO; the gradients are returned in the pre-RoPE frame (R^T at each row's
    position).  With branch_k / branch_v ([P, Lq, Hkv, D], the chunk's own keys and
    values of every pass) the branch keys of passes 2..p at the row's own position add
    their part to dq and give dk_b, dv_b (the chunk's branch-pass gradients; pass 1
    zero).  Summed over the ring's pairs these give the whole sequence's gradients.

    qc [P, Lq, H, D], doc [P, Lq, H, D]; kt, vt [Lk, Hkv, D]; lse_c, delta_c [P, H, Lq].
    Returns (dq [P, Lq, H, D], dk [Lk, Hkv, D], dv [Lk, Hkv, D], dk_b, dv_b or None)."""
    P, Lq, H, D = qc.shape
    Lk, Hkv = kt.shape[0], kt.shape[1]
    g = H // Hkv
    sc = _scale(D, scale)
    ktr = rope_rotate(kt.astype(np.float64), np.arange(Lk) + kv_start, theta)
    qr = np.stack([rope_rotate(qc[p0].astype(np.float64), np.arange(Lq) + q_start + p0, theta) for p0 in range(P)])
    kbr = None
    if branch_k is not None:
        kbr = np.stack([rope_rotate(branch_k[j].astype(np.float64), np.arange(Lq) + q_start + j, theta)
                        for j in range(P)])
    if rope_round == "bf16":
        ktr, qr = bf16_round(ktr), bf16_round(qr)
        if kbr is not None:
            kbr = bf16_round(kbr)
    visible = (kv_start + np.arange(Lk))[None, :] <= (q_start + np.arange(Lq))[:, None]
    vt64 = vt.astype(np.float64)
    dqr = np.zeros((P, Lq, H, D))
    dkr = np.zeros((Lk, Hkv, D))
    dv = np.zeros((Lk, Hkv, D))
    dkbr = np.zeros((P, Lq, Hkv, D)) if kbr is not None else None
    dvb = np.zeros((P, Lq, Hkv, D)) if kbr is not None else None
    for h in range(H):
        kv = h // g
        for p0 in range(P):
            l = lse_c[p0, h][:, None]
            dl = delta_c[p0, h][:, None]
            do = doc[p0, :, h].astype(np.float64)
            s = np.where(visible, sc * (qr[p0, :, h] @ ktr[:, kv].T), -np.inf)
            Pm = np.exp(s - l)
            dS = Pm * (do @ vt64[:, kv].T - dl)
            dqr[p0, :, h] += sc * dS @ ktr[:, kv]
            dkr[:, kv] += sc * dS.T @ qr[p0, :, h]
            dv[:, kv] += Pm.T @ do
            if kbr is not None:
                for j in range(1, p0 + 1):
                    sb = sc * np.sum(qr[p0, :, h] * kbr[j, :, kv], axis=1, keepdims=True)
                    pb = np.exp(sb - l)
                    dsb = pb * (np.sum(do * branch_v[j, :, kv].astype(np.float64), axis=1, keepdims=True) - dl)
                    dqr[p0, :, h] += sc * dsb * kbr[j, :, kv]
                    dkbr[j, :, kv] += sc * dsb * qr[p0, :, h]
                    dvb[j, :, kv] += pb * do
    dq = np.stack([rope_rotate(dqr[p0], np.arange(Lq) + q_start + p0, theta, inverse=True) for p0 in range(P)])
    dk = rope_rotate(dkr, np.arange(Lk) + kv_start, theta, inverse=True)
    if kbr is not None:
        dkb = np.stack([rope_rotate(dkbr[j], np.arange(Lq) + q_start + j, theta, inverse=True) for j in range(P)])
        return dq, dk, dv, dkb, dvb
    return dq, dk, dv, None, None
