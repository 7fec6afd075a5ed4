"""Comparing the CUDA block-draft attention with its fp64 oracle (test code only)."""

from __future__ import annotations

import numpy as np
import torch

import ttt_inputs
from oracle import block_draft_oracle as bd
from tests.parity import GRAD_REL_L2, LSE_MAX_ABS, O_MAX_ABS, rel_l2, to64


def gpu_tensors(w: ttt_inputs.BlockWorkload, inp: ttt_inputs.BlockInputs, device="cuda"):
    """Inputs on the device in the public layout of the workload, plus the packed
    keyword arguments."""
    t = {n: getattr(inp, n).to(device) for n in ("k_ctx", "v_ctx", "qb", "kb", "vb", "do", "anchors")}
    kw = {}
    if w.dense:
        B, S, nblk = w.nseq, w.ctx_lengths[0], w.nblocks[0]
        for n in ("k_ctx", "v_ctx"):
            t[n] = t[n].view(B, S, *t[n].shape[1:])
        for n in ("qb", "kb", "vb", "do"):
            t[n] = t[n].view(B, nblk, *t[n].shape[1:])
        t["anchors"] = t["anchors"].view(B, nblk)
    else:
        kw = dict(cu_ctx=torch.tensor(w.cu_ctx, dtype=torch.int32, device=device),
                  cu_blocks=torch.tensor(w.cu_blocks, dtype=torch.int32, device=device),
                  max_ctx=max(w.ctx_lengths), max_blocks=max(w.nblocks))
    return {n: x.contiguous() for n, x in t.items()}, kw


def run_gpu(w, inp, with_grad=True, scale=None, reuse_rotation=False, deterministic=False, window=0):
    from attention_pass_rope_b200 import ops
    t, kw = gpu_tensors(w, inp)
    args = (t["k_ctx"], t["v_ctx"], t["qb"], t["kb"], t["vb"], t["anchors"])
    ws = None
    if reuse_rotation:
        lay = ops._block_layout(*args, kw.get("cu_ctx"), kw.get("cu_blocks"), kw.get("max_ctx"),
                                kw.get("max_blocks"))
        ws = ops.alloc_workspace(ops.block_workspace_bytes(lay, t["anchors"], w.theta, scale, for_backward=True),
                                 t["qb"].device)
    o, lse = ops.block_attn_fwd(*args, theta=w.theta, scale=scale, workspace=ws, window=window, **kw)
    out = {"o": o.reshape(w.NB, w.Bs, w.H, w.D), "lse": lse}
    if with_grad:
        g = ops.block_attn_bwd(*args, o, lse, t["do"], theta=w.theta, scale=scale, workspace=ws,
                               rotated_in_workspace=reuse_rotation, deterministic=deterministic, window=window,
                               **kw)
        out.update(dk_ctx=g[0].reshape(w.Tc, w.Hkv, w.D), dv_ctx=g[1].reshape(w.Tc, w.Hkv, w.D),
                   dqb=g[2].reshape(w.NB, w.Bs, w.H, w.D), dkb=g[3].reshape(w.NB, w.Bs, w.Hkv, w.D),
                   dvb=g[4].reshape(w.NB, w.Bs, w.Hkv, w.D))
    torch.cuda.synchronize()
    return out


def gpu_lse_rows(w, lse, n, h):
    """lse of sequence n's block rows for head h, from the public layout."""
    if w.dense:
        return lse[n, h]
    b0, b1 = w.cu_blocks[n], w.cu_blocks[n + 1]
    return lse[h, b0 * w.Bs: b1 * w.Bs]


def compare(w, inp, gpu, with_grad=True, kv_heads=None, seqs=None, scale=None, window=0):
    """Oracle (rope_round="bf16") per sequence and KV-head group; element-wise metrics."""
    g = w.H // w.Hkv
    kv_heads = range(w.Hkv) if kv_heads is None else kv_heads
    seqs = range(w.nseq) if seqs is None else seqs
    o_err, l_err = 0.0, 0.0
    pairs = {n: ([], []) for n in ("dqb", "dk_ctx", "dv_ctx", "dkb", "dvb")}
    f64 = lambda x: x.float().numpy().astype(np.float64)
    for n in seqs:
        c0, c1 = w.cu_ctx[n], w.cu_ctx[n + 1]
        b0, b1 = w.cu_blocks[n], w.cu_blocks[n + 1]
        if b1 == b0 or c1 == c0:
            continue
        anchors = inp.anchors[b0:b1].tolist()
        for kv in kv_heads:
            hs = slice(kv * g, (kv + 1) * g)
            ks = slice(kv, kv + 1)
            c = dict(k_ctx=f64(inp.k_ctx[c0:c1, ks]), v_ctx=f64(inp.v_ctx[c0:c1, ks]), anchors=anchors,
                     qb=f64(inp.qb[b0:b1, :, hs]), kb=f64(inp.kb[b0:b1, :, ks]), vb=f64(inp.vb[b0:b1, :, ks]))
            O, lse = bd.forward_twopart(theta=w.theta, scale=scale, rope_round="bf16", window=window, **c)
            o_err = max(o_err, float(np.max(np.abs(to64(gpu["o"][b0:b1, :, hs]) - O))))
            for hh in range(g):
                got = to64(gpu_lse_rows(w, gpu["lse"], n, kv * g + hh))
                l_err = max(l_err, float(np.max(np.abs(got - lse[:, hh].reshape(-1)))))
            if with_grad:
                ref = bd.backward_twopart(do=f64(inp.do[b0:b1, :, hs]), O=O, lse=lse, theta=w.theta, scale=scale,
                                          rope_round="bf16", window=window, **c)
                got = (gpu["dqb"][b0:b1, :, hs], gpu["dk_ctx"][c0:c1, ks], gpu["dv_ctx"][c0:c1, ks],
                       gpu["dkb"][b0:b1, :, ks], gpu["dvb"][b0:b1, :, ks])
                for name, r_, g_ in zip(("dqb", "dk_ctx", "dv_ctx", "dkb", "dvb"), ref, got):
                    assert torch.isfinite(g_.float()).all(), name
                    pairs[name][0].append(to64(g_).ravel())
                    pairs[name][1].append(r_.ravel())
    m = {"o_max_abs": o_err, "lse_max_abs": l_err}
    if with_grad:
        for name, (got, ref) in pairs.items():
            if got:
                m[name + "_rel_l2"] = rel_l2(np.concatenate(got), np.concatenate(ref))
    return m


def assert_within(m):
    assert m["o_max_abs"] <= O_MAX_ABS, m
    assert m["lse_max_abs"] <= LSE_MAX_ABS, m
    for k, v in m.items():
        if k.endswith("_rel_l2"):
            assert v <= GRAD_REL_L2, (k, m)
