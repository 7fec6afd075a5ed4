"""fp64 CPU oracle for the soft cross-entropy distillation loss of the TTT draft passes.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, the package's smoke check and the bench's
CPU baseline may import this module; no library code does, and it shares no code with
any CUDA path.

What is computed (source, by page and section):

* "DFlash/DSpark and EAGLE-3 TTT draft co-training for speculative decoding
  (Megatron backend)" (NeMo-RL issue 3698), section "What I'm working on", item 3:
  the draft is trained with a soft cross-entropy (distillation) loss against the
  target, computed in token chunks and split over the vocabulary, normalised per
  pass (per block slot for block drafters) over the whole global batch.  Item 2:
  the draft rides the target's live head (it has no lm_head of its own).
* "bounded multi-pass EAGLE-3 TTT provider" (NeMo-RL PR 3725), merge note 3: the
  loss takes a ``token_chunk_size`` (default 4096 tokens).

The pages name the loss and nothing of its formula.  Readings where they are silent:

* Draft logits of pass p at token t: z = W h_{p,t}, W [V, d] the vocabulary head,
  h_{p,t} the draft's last hidden state; no bias.
* The teacher is the target's logits y; its distribution is q = softmax(y) at
  temperature 1.  The teacher is not differentiated.
* Alignment: pass p (p = 1..P) at token t learns the teacher row of position
  t + p - 1 of the same sequence.  Pass 1 learns the row of its own position, and
  each later pass predicts one more token ahead (the shift that the passes' RoPE
  positions i + p - 1 carry).  A pair whose teacher position lies past the end of
  its sequence, or has loss mask 0, is invalid: loss 0, no gradient.
* Loss of a valid pair: l = logsumexp(z) - sum_v q_v z_v, the cross-entropy of
  softmax(z) against q.
* Per-pass normalisation: L_p = w_p / N_p * sum_t l_{p,t}, N_p the number of valid
  pairs of pass p ("global": a caller may pass counts summed over ranks instead);
  N_p = 0 gives L_p = 0.  Total L = sum_p L_p; w_p defaults to 1.
* Gradients of g * L: dz = g * w_p / N_p * (softmax(z) - q) for a valid pair,
  dh = W^T dz, dW = sum over pairs of dz h^T.
* The token chunk size changes only the order in which an implementation visits the
  pairs, not the values; the oracle takes all pairs at once.

* Per-slot normalisation (same item): block drafters normalise per slot of a block
  instead of per pass.  The general form takes, for every draft row, its teacher
  position (or -1) and its normalisation group: L_g = w_g / N_g * sum over the valid
  rows of group g, L = sum_g L_g.  The TTT passes are the case group = pass, teacher =
  t + p - 1 (:func:`ttt_mapping`).

Array conventions: h [P, T, d] (pass-major, tokens of all sequences concatenated,
``cu_seqlens`` their boundaries); W [V, d]; y [T, V]; loss_mask [T] (teacher
positions), 1 = counted.  The general form: draft rows h [R, d], y [Ty, V], loss_mask
[Ty], teacher [R], group [R].  Inputs are taken as given (bf16 values in fp64).
"""

from __future__ import annotations

import numpy as np


def teacher_index(cu_seqlens, P, loss_mask=None):
    """[P, T] int64: the teacher position of each (pass, token) pair, -1 if invalid."""
    cu = [int(c) for c in cu_seqlens]
    T = cu[-1]
    idx = np.full((P, T), -1, dtype=np.int64)
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        for p in range(1, P + 1):
            for t in range(a, b):
                u = t + p - 1
                if u < b and (loss_mask is None or loss_mask[u]):
                    idx[p - 1, t] = u
    return idx


def _logsumexp(x, axis=-1):
    m = np.max(x, axis=axis, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    return np.squeeze(m, axis) + np.log(np.sum(np.exp(x - m), axis=axis))


def _softmax(x):
    e = np.exp(x - np.max(x, axis=-1, keepdims=True))
    return e / np.sum(e, axis=-1, keepdims=True)


def _f64(a):
    return np.asarray(a.float().numpy() if hasattr(a, "float") else a, dtype=np.float64)


def pair_loss(z, yrow):
    """Loss of one valid pair from its draft logits z [V] and teacher logits yrow [V]."""
    z = np.asarray(z, dtype=np.float64)
    q = _softmax(np.asarray(yrow, dtype=np.float64))
    return float(_logsumexp(z) - np.dot(q, z))


def pass_counts(idx, counts=None):
    """N_p: the given counts, else the number of valid pairs of each pass."""
    if counts is not None:
        return np.asarray(counts, dtype=np.float64)
    return (idx >= 0).sum(axis=1).astype(np.float64)


def forward(h, W, y, cu_seqlens, loss_mask=None, pass_weight=None, counts=None):
    """The loss.  Returns a dict: ``rows`` [P, T] (l of each pair, 0 if invalid),
    ``lse_z`` [P, T], ``pass_loss`` [P], ``loss`` (scalar), ``counts`` [P]."""
    h, W, y = _f64(h), _f64(W), _f64(y)
    P, T, _ = h.shape
    idx = teacher_index(cu_seqlens, P, loss_mask)
    z = h @ W.T                                   # [P, T, V]
    lse_z = _logsumexp(z)
    rows = np.zeros((P, T))
    for p in range(P):
        for t in range(T):
            u = idx[p, t]
            if u >= 0:
                rows[p, t] = pair_loss(z[p, t], y[u])
    w = np.ones(P) if pass_weight is None else np.asarray(pass_weight, dtype=np.float64)
    n = pass_counts(idx, counts)
    pass_loss = np.array([w[p] / n[p] * rows[p].sum() if n[p] > 0 else 0.0 for p in range(P)])
    return {"rows": rows, "lse_z": lse_z, "pass_loss": pass_loss, "loss": float(pass_loss.sum()), "counts": n}


def logit_grad(h, W, y, cu_seqlens, loss_mask=None, pass_weight=None, counts=None, grad=1.0):
    """dz [P, T, V]: the gradient of grad * L with respect to the draft logits."""
    h, W, y = _f64(h), _f64(W), _f64(y)
    P, T, _ = h.shape
    idx = teacher_index(cu_seqlens, P, loss_mask)
    w = np.ones(P) if pass_weight is None else np.asarray(pass_weight, dtype=np.float64)
    n = pass_counts(idx, counts)
    z = h @ W.T
    dz = np.zeros_like(z)
    for p in range(P):
        if n[p] <= 0:
            continue
        for t in range(T):
            u = idx[p, t]
            if u >= 0:
                dz[p, t] = grad * w[p] / n[p] * (_softmax(z[p, t]) - _softmax(y[u]))
    return dz


def backward(h, W, y, cu_seqlens, loss_mask=None, pass_weight=None, counts=None, grad=1.0):
    """(dh [P, T, d], dW [V, d]) of grad * L."""
    dz = logit_grad(h, W, y, cu_seqlens, loss_mask, pass_weight, counts, grad)
    h, W = _f64(h), _f64(W)
    dh = dz @ W
    dW = dz.reshape(-1, dz.shape[-1]).T @ h.reshape(-1, h.shape[-1])
    return dh, dW


def row_forward(h_row, W, y_row):
    """Loss and logsumexp of one valid pair, from its hidden state alone (large shapes)."""
    z = _f64(W) @ _f64(h_row)
    return pair_loss(z, _f64(y_row)), float(_logsumexp(z))


def row_dh(h_row, W, y_row, coef):
    """dh of one valid pair whose gradient coefficient (grad * w_p / N_p) is ``coef``."""
    W = _f64(W)
    z = W @ _f64(h_row)
    return coef * ((_softmax(z) - _softmax(_f64(y_row))) @ W)


def rows_logits(h_rows, W, slice_rows=16384):
    """z [n, V] of a few draft rows h_rows [n, d] (fp64).  W is converted to fp64 a slice
    of vocabulary rows at a time, so that a full-size head is never held in fp64; each
    logit is the same dot product as in :func:`forward`."""
    H = _f64(h_rows)
    V = W.shape[0]
    z = np.empty((H.shape[0], V))
    for v0 in range(0, V, slice_rows):
        Ws = _f64(W[v0:v0 + slice_rows])
        z[:, v0:v0 + Ws.shape[0]] = H @ Ws.T
    return z


def rows_forward(h_rows, W, y_rows):
    """(loss [n], lse [n]) of n valid pairs from their hidden states and teacher rows."""
    z = rows_logits(h_rows, W)
    y = _f64(y_rows)
    loss = np.array([pair_loss(z[i], y[i]) for i in range(z.shape[0])])
    return loss, _logsumexp(z)


def rows_dh(h_rows, W, y_rows, coef, slice_rows=16384):
    """dh [n, d] of n valid pairs with gradient coefficients coef [n] (grad * w_p / N_p)."""
    z = rows_logits(h_rows, W, slice_rows)
    dz = np.asarray(coef, dtype=np.float64)[:, None] * (_softmax(z) - _softmax(_f64(y_rows)))
    V = W.shape[0]
    dh = np.zeros((z.shape[0], W.shape[1]))
    for v0 in range(0, V, slice_rows):
        Ws = _f64(W[v0:v0 + slice_rows])
        dh += dz[:, v0:v0 + Ws.shape[0]] @ Ws
    return dh


def ttt_mapping(cu_seqlens, P):
    """(teacher [P*T], group [P*T]) of the TTT passes in the general form: row p*T + t
    learns position t + p of its sequence (or nothing), in group p."""
    idx = teacher_index(cu_seqlens, P)
    T = idx.shape[1]
    return idx.reshape(-1), np.repeat(np.arange(P), T)


def forward_mapped(h_rows, W, y, teacher, group, ngroups, loss_mask=None, group_weight=None, counts=None):
    """The loss with an explicit teacher position and normalisation group per draft row.
    Returns a dict: ``rows`` [R], ``lse_z`` [R], ``group_loss`` [G], ``loss``, ``counts`` [G]."""
    h, W, y = _f64(h_rows), _f64(W), _f64(y)
    teacher = np.asarray(teacher, dtype=np.int64)
    group = np.asarray(group, dtype=np.int64)
    Ty = y.shape[0]
    valid = (teacher >= 0) & (teacher < Ty)
    if loss_mask is not None:
        m = np.asarray(loss_mask).astype(bool)
        valid &= np.array([bool(m[u]) if 0 <= u < Ty else False for u in teacher])
    z = h @ W.T
    lse_z = _logsumexp(z)
    rows = np.zeros(h.shape[0])
    for r in np.nonzero(valid)[0]:
        rows[r] = pair_loss(z[r], y[teacher[r]])
    w = np.ones(ngroups) if group_weight is None else np.asarray(group_weight, dtype=np.float64)
    n = (np.array([np.sum(valid & (group == g)) for g in range(ngroups)], dtype=np.float64)
         if counts is None else np.asarray(counts, dtype=np.float64))
    gl = np.array([w[g] / n[g] * rows[group == g].sum() if n[g] > 0 else 0.0 for g in range(ngroups)])
    return {"rows": rows, "lse_z": lse_z, "group_loss": gl, "loss": float(gl.sum()), "counts": n, "valid": valid}


def backward_mapped(h_rows, W, y, teacher, group, ngroups, loss_mask=None, group_weight=None, counts=None,
                    grad=1.0):
    """(dh [R, d], dW [V, d]) of grad * L in the general form."""
    out = forward_mapped(h_rows, W, y, teacher, group, ngroups, loss_mask, group_weight, counts)
    h, W, y = _f64(h_rows), _f64(W), _f64(y)
    teacher = np.asarray(teacher, dtype=np.int64)
    group = np.asarray(group, dtype=np.int64)
    w = np.ones(ngroups) if group_weight is None else np.asarray(group_weight, dtype=np.float64)
    n = out["counts"]
    z = h @ W.T
    dz = np.zeros_like(z)
    for r in np.nonzero(out["valid"])[0]:
        g = group[r]
        if n[g] > 0:
            dz[r] = grad * w[g] / n[g] * (_softmax(z[r]) - _softmax(y[teacher[r]]))
    return dz @ W, dz.T @ h
