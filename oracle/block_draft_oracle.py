"""fp64 CPU oracle for the block-draft attention of DFlash/DSpark drafters.

TEST INFRASTRUCTURE ONLY.  Only ``tests/`` may import this module; no library code
does, and it shares no code with any CUDA path.

What is computed (source, by page and section):

* "DFlash/DSpark and EAGLE-3 TTT draft co-training for speculative decoding
  (Megatron backend)" (NeMo-RL issue 3698), section "What I'm working on",
  item 2: block drafters draft a block made of an anchor and mask tokens, with
  bidirectional attention inside the block and the trunk truncated at the
  anchor.  Item 4: the same attention on the packed (THD) layout.

The page gives the pattern in one line.  Readings where it is silent:

* A block of Bs draft tokens starts at an anchor position a of the sequence:
  the anchor and Bs - 1 mask tokens, at positions a, a+1, ..., a+Bs-1; each has
  its own query, key and value.
* The trunk of a block is the context keys and values at positions 0..a: causal
  up to and including the anchor ("truncated at the anchor").
* Every query of the block sees that trunk and all Bs keys of its own block
  (bidirectional), nothing of other blocks.  The two parts are merged exactly
  through their log-sum-exps, as in the TTT trunk+branch attention.
* RoPE is rotate-half at the token's position (trunk key t at t, block token j
  at a+j), the same frequencies as the TTT attention; the softmax scale is
  1/sqrt(D) unless given; query head h reads KV head h // (H // Hkv).
* Sliding-window block layers (item 4 of the same list names them) see only the
  last ``window`` context positions of their trunk: t in [max(0, a - window + 1), a].
  The page names the layers and nothing more; the window reading here is the plainest
  one that keeps the anchor as the trunk's end.  ``window=None`` (or 0) is the full
  trunk 0..a.
* ``rope_round="bf16"`` rounds the rotated queries and keys to bf16 (round to
  nearest even) before the dot products, the library's defined semantics for
  this attention as for the TTT attention (bf16 operands into the tensor cores);
  the default ``None`` keeps them exact.  Gradients treat the rounding as the
  identity.

Array conventions (one sequence): trunk k_ctx, v_ctx [L, Hkv, D]; anchors [nb]
(ints in 0..L-1); block qb [nb, Bs, H, D], kb, vb [nb, Bs, Hkv, D].  Outputs:
O [nb, Bs, H, D], lse [nb, H, Bs].

Two forms that share nothing but the RoPE helper and the input arrays:

* :func:`forward_bruteforce` / :func:`backward_bruteforce`: the L trunk keys and
  all nb*Bs block keys concatenated, an explicit boolean mask, one softmax.
* :func:`forward_twopart` / :func:`backward_twopart`: a trunk softmax over t <= a
  and a block softmax over the Bs block keys, merged by
  lse = logaddexp(lse_trunk, lse_block).
"""

from __future__ import annotations

import math

import numpy as np

from oracle.ttt_oracle import bf16_round, rope_rotate


def _scale(D, scale):
    return 1.0 / math.sqrt(D) if scale is None else float(scale)


def _rotate(k_ctx, anchors, qb, kb, theta, pos_offset=0, rope_round=None):
    """RoPE at the tokens' positions: trunk key t at t, block token j at anchor + j;
    ``rope_round="bf16"`` rounds the rotated arrays to bf16."""
    L = k_ctx.shape[0]
    nb, Bs = qb.shape[:2]
    kt = rope_rotate(k_ctx, np.arange(L) + pos_offset, theta)
    pos_b = (np.asarray(anchors)[:, None] + np.arange(Bs)[None, :] + pos_offset).reshape(-1)
    qr = rope_rotate(qb.reshape(nb * Bs, *qb.shape[2:]), pos_b, theta).reshape(qb.shape)
    kr = rope_rotate(kb.reshape(nb * Bs, *kb.shape[2:]), pos_b, theta).reshape(kb.shape)
    if rope_round == "bf16":
        kt, qr, kr = bf16_round(kt), bf16_round(qr), bf16_round(kr)
    elif rope_round is not None:
        raise ValueError(rope_round)
    return kt, qr, kr


def trunk_start(a, window):
    """First trunk key of a block anchored at a: 0, or a - window + 1 (at least 0) for a
    sliding-window layer."""
    return 0 if not window else max(0, a - int(window) + 1)


def block_mask(L, anchors, Bs, window=None):
    """[nb*Bs, L + nb*Bs] visibility: block query (b, j) sees trunk t in
    [trunk_start(anchor_b), anchor_b] and the Bs keys of block b."""
    nb = len(anchors)
    m = np.zeros((nb * Bs, L + nb * Bs), dtype=bool)
    for b, a in enumerate(anchors):
        rows = slice(b * Bs, (b + 1) * Bs)
        m[rows, trunk_start(a, window): a + 1] = True
        m[rows, L + b * Bs: L + (b + 1) * Bs] = True
    return m


def forward_bruteforce(k_ctx, v_ctx, anchors, qb, kb, vb, theta, scale=None, pos_offset=0, rope_round=None,
                       window=None):
    L, Hkv, D = k_ctx.shape
    nb, Bs, H, _ = qb.shape
    g = H // Hkv
    sc = _scale(D, scale)
    kt, qr, kr = _rotate(k_ctx, anchors, qb, kb, theta, pos_offset, rope_round)
    K = np.concatenate([kt, kr.reshape(nb * Bs, Hkv, D)])      # [L + nb*Bs, Hkv, D]
    V = np.concatenate([v_ctx, vb.reshape(nb * Bs, Hkv, D)])
    Q = qr.reshape(nb * Bs, H, D)
    m = block_mask(L, anchors, Bs, window)
    O = np.zeros((nb * Bs, H, D))
    lse = np.zeros((H, nb * Bs))
    for h in range(H):
        S = sc * (Q[:, h] @ K[:, h // g].T)
        S = np.where(m, S, -np.inf)
        mx = S.max(axis=1, keepdims=True)
        E = np.exp(S - mx)
        s = E.sum(axis=1, keepdims=True)
        O[:, h] = (E / s) @ V[:, h // g]
        lse[h] = (mx + np.log(s))[:, 0]
    return O.reshape(nb, Bs, H, D), lse.reshape(H, nb, Bs).transpose(1, 0, 2)


def backward_bruteforce(k_ctx, v_ctx, anchors, qb, kb, vb, do, theta, scale=None, pos_offset=0,
                        rope_round=None, window=None):
    """Gradients with respect to the pre-RoPE inputs: (dqb, dk_ctx, dv_ctx, dkb, dvb)."""
    L, Hkv, D = k_ctx.shape
    nb, Bs, H, _ = qb.shape
    g = H // Hkv
    sc = _scale(D, scale)
    kt, qr, kr = _rotate(k_ctx, anchors, qb, kb, theta, pos_offset, rope_round)
    K = np.concatenate([kt, kr.reshape(nb * Bs, Hkv, D)])
    V = np.concatenate([v_ctx, vb.reshape(nb * Bs, Hkv, D)])
    Q = qr.reshape(nb * Bs, H, D)
    dO = do.reshape(nb * Bs, H, D)
    m = block_mask(L, anchors, Bs, window)
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    for h in range(H):
        kv = h // g
        S = np.where(m, sc * (Q[:, h] @ K[:, kv].T), -np.inf)
        Pm = np.exp(S - S.max(axis=1, keepdims=True))
        Pm /= Pm.sum(axis=1, keepdims=True)
        O = Pm @ V[:, kv]
        dP = dO[:, h] @ V[:, kv].T
        dS = Pm * (dP - np.sum(dO[:, h] * O, axis=1, keepdims=True))
        dQ[:, h] = sc * dS @ K[:, kv]
        dK[:, kv] += sc * dS.T @ Q[:, h]
        dV[:, kv] += Pm.T @ dO[:, h]
    pos_b = (np.asarray(anchors)[:, None] + np.arange(Bs)[None, :] + pos_offset).reshape(-1)
    dqb = rope_rotate(dQ, pos_b, theta, inverse=True).reshape(qb.shape)
    dk_ctx = rope_rotate(dK[:L], np.arange(L) + pos_offset, theta, inverse=True)
    dkb = rope_rotate(dK[L:], pos_b, theta, inverse=True).reshape(kb.shape)
    return dqb, dk_ctx, dV[:L], dkb, dV[L:].reshape(vb.shape)


def forward_twopart(k_ctx, v_ctx, anchors, qb, kb, vb, theta, scale=None, pos_offset=0, return_parts=False,
                    rope_round=None, window=None):
    """Per block: trunk softmax over its trunk keys (t <= anchor, from trunk_start), block
    softmax over its Bs keys, merged."""
    L, Hkv, D = k_ctx.shape
    nb, Bs, H, _ = qb.shape
    g = H // Hkv
    sc = _scale(D, scale)
    kt, qr, kr = _rotate(k_ctx, anchors, qb, kb, theta, pos_offset, rope_round)
    O = np.zeros((nb, Bs, H, D))
    lse = np.zeros((nb, H, Bs))
    parts = []
    for b, a in enumerate(anchors):
        t0 = trunk_start(a, window)
        for h in range(H):
            kv = h // g
            St = sc * (qr[b, :, h] @ kt[t0: a + 1, kv].T)      # [Bs, a+1-t0]
            mt = St.max(axis=1, keepdims=True)
            Et = np.exp(St - mt)
            lt = mt[:, 0] + np.log(Et.sum(axis=1))
            Ot = (Et @ v_ctx[t0: a + 1, kv]) / Et.sum(axis=1, keepdims=True)
            Sb = sc * (qr[b, :, h] @ kr[b, :, kv].T)           # [Bs, Bs], bidirectional
            mb = Sb.max(axis=1, keepdims=True)
            Eb = np.exp(Sb - mb)
            lb = mb[:, 0] + np.log(Eb.sum(axis=1))
            Ob = (Eb @ vb[b, :, kv]) / Eb.sum(axis=1, keepdims=True)
            l = np.logaddexp(lt, lb)
            O[b, :, h] = np.exp(lt - l)[:, None] * Ot + np.exp(lb - l)[:, None] * Ob
            lse[b, h] = l
            parts.append((b, h, lt, lb))
    return (O, lse, parts) if return_parts else (O, lse)


def backward_twopart(k_ctx, v_ctx, anchors, qb, kb, vb, do, O, lse, theta, scale=None, pos_offset=0,
                     rope_round=None, window=None):
    """Gradients from the merged lse: P = exp(s - lse) for both parts,
    delta = rowsum(dO * O), dS = P (dP - delta)."""
    L, Hkv, D = k_ctx.shape
    nb, Bs, H, _ = qb.shape
    g = H // Hkv
    sc = _scale(D, scale)
    kt, qr, kr = _rotate(k_ctx, anchors, qb, kb, theta, pos_offset, rope_round)
    dqr = np.zeros_like(qr)
    dkt = np.zeros_like(kt)
    dvt = np.zeros_like(v_ctx)
    dkr = np.zeros_like(kr)
    dvb = np.zeros_like(vb)
    for b, a in enumerate(anchors):
        t0 = trunk_start(a, window)
        for h in range(H):
            kv = h // g
            l = lse[b, h][:, None]
            delta = np.sum(do[b, :, h] * O[b, :, h], axis=1, keepdims=True)
            Pt = np.exp(sc * (qr[b, :, h] @ kt[t0: a + 1, kv].T) - l)
            dSt = Pt * (do[b, :, h] @ v_ctx[t0: a + 1, kv].T - delta)
            Pb = np.exp(sc * (qr[b, :, h] @ kr[b, :, kv].T) - l)
            dSb = Pb * (do[b, :, h] @ vb[b, :, kv].T - delta)
            dqr[b, :, h] = sc * (dSt @ kt[t0: a + 1, kv] + dSb @ kr[b, :, kv])
            dkt[t0: a + 1, kv] += sc * dSt.T @ qr[b, :, h]
            dvt[t0: a + 1, kv] += Pt.T @ do[b, :, h]
            dkr[b, :, kv] += sc * dSb.T @ qr[b, :, h]
            dvb[b, :, kv] += Pb.T @ do[b, :, h]
    pos_b = (np.asarray(anchors)[:, None] + np.arange(Bs)[None, :] + pos_offset).reshape(-1)
    dqb = rope_rotate(dqr.reshape(nb * Bs, H, D), pos_b, theta, inverse=True).reshape(qb.shape)
    dk_ctx = rope_rotate(dkt, np.arange(L) + pos_offset, theta, inverse=True)
    dkb = rope_rotate(dkr.reshape(nb * Bs, Hkv, D), pos_b, theta, inverse=True).reshape(kb.shape)
    return dqb, dk_ctx, dvt, dkb, dvb
