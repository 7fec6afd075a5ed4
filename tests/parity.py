"""Helpers for comparing the CUDA path with the fp64 oracle (test code only)."""

from __future__ import annotations

import numpy as np
import torch

import ttt_inputs
from oracle import ttt_oracle as orc

# Tolerances from the method's accuracy statement: bf16 inputs, fp32 accumulation.
O_MAX_ABS = 2e-2
LSE_MAX_ABS = 1e-3
GRAD_REL_L2 = 1e-2


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    a = a.ravel()
    b = b.ravel()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def gpu_shapes(w: ttt_inputs.Workload, inp: ttt_inputs.Inputs, device="cuda"):
    """Move inputs to the device in the public layout of the workload."""
    def dev(t):
        if t is None:
            return None
        t = t.to(device)
        if w.dense:
            B, S = len(w.lengths), w.lengths[0]
            t = t.view(t.shape[0], B, S, *t.shape[2:])
        return t.contiguous()
    cu = None
    if not w.dense:
        cu = torch.tensor(w.cu_seqlens, dtype=torch.int32, device=device)
    return dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.do), cu


def flat(t: torch.Tensor, w) -> torch.Tensor:
    """[P, B, S, ...] -> [P, T, ...] (dense); packed tensors unchanged."""
    if w.dense:
        return t.reshape(t.shape[0], -1, *t.shape[3:])
    return t


def run_gpu(w, inp, with_grad=True, reuse_rotation=False, scale=None):
    """Forward (+ backward) through the C ABI.  ``reuse_rotation``: one workspace for
    both calls and the backward told to reuse the forward's rotated q~ / k~.
    ``scale``: softmax scale passed to the library (None: its default 1/sqrt(D))."""
    from attention_pass_rope_b200 import ops, ttt_attn_bwd, ttt_attn_fwd
    q, k, v, do, cu = gpu_shapes(w, inp)
    kw = dict(theta=w.theta, scale=scale, cu_seqlens=cu, max_seqlen=None if w.dense else w.max_seqlen)
    ws = None
    if reuse_rotation:
        lay = ops._layout(q, k, v, cu, kw["max_seqlen"])
        ws = ops.alloc_workspace(ops.workspace_bytes(lay, w.theta, scale, for_backward=True), q.device)
    o, lse = ttt_attn_fwd(q, k, v, workspace=ws, **kw)
    out = {"o": flat(o, w), "lse": lse}
    if with_grad:
        dq, dk, dv = ttt_attn_bwd(q, k, v, o, lse, do, workspace=ws, rotated_in_workspace=reuse_rotation, **kw)
        out.update(dq=flat(dq, w), dk=flat(dk, w), dv=flat(dv, w))
    torch.cuda.synchronize()
    return out


def oracle_np(inp):
    return tuple(to64(t) if t is not None else None for t in (inp.q, inp.k, inp.v, inp.do))


def per_pass_rel_l2(got: np.ndarray, ref: np.ndarray):
    """Relative L2 error of each pass ([P, T, heads, D] arrays; NaN entries of ``ref``
    are outside the sampled subset and skipped), and the worst (pass, head) pair.

    The whole-tensor figure is dominated by the pass with the largest gradient (pass 1
    carries every trunk key's gradient), so an error confined to the branch passes
    would be diluted in it; each pass is therefore also held to the bound on its own."""
    per_pass = []
    worst = (0.0, None)
    for p in range(ref.shape[0]):
        s = ~np.isnan(ref[p])
        if not s.any() or np.linalg.norm(ref[p][s]) == 0.0:
            per_pass.append(None)
            continue
        per_pass.append(rel_l2(got[p][s], ref[p][s]))
        for h in range(ref.shape[2]):
            sh = ~np.isnan(ref[p, :, h])
            if sh.any() and np.linalg.norm(ref[p, :, h][sh]) > 0.0:
                e = rel_l2(got[p, :, h][sh], ref[p, :, h][sh])
                if e > worst[0]:
                    worst = (e, (p, h))
    return per_pass, worst


def compare_full(w, inp, gpu, with_grad=True, kv_heads=None, seqs=None, scale=None):
    """Oracle on (a subset of) the workload, element-wise comparison.  Returns metrics:
    O and lse max-abs, dq/dk/dv relative L2 over the whole tensor and per pass, and the
    worst (pass, head) relative L2 of each gradient."""
    q, k, v, do = oracle_np(inp)
    cu = w.cu_seqlens
    heads = None
    if kv_heads is not None:
        g = w.H // w.Hkv
        heads = [h for kv in kv_heads for h in range(kv * g, (kv + 1) * g)]
    O, lse = orc.forward_packed(q, k, v, cu, w.theta, w.dense, scale=scale, heads=heads, seqs=seqs)
    m = {}
    Og = to64(gpu["o"])
    lg = to64(gpu["lse"])
    sel = ~np.isnan(O)
    m["o_max_abs"] = float(np.max(np.abs(Og[sel] - O[sel])))
    sl = ~np.isnan(lse)
    m["lse_max_abs"] = float(np.max(np.abs(lg[sl] - lse[sl])))
    assert np.all(np.isfinite(Og)) and np.all(np.isfinite(lg))
    if with_grad:
        # rows outside the sampled subset are NaN in the oracle lse and never read
        dq, dk, dv = orc.backward_packed(q, k, v, do, lse, cu, w.theta, w.dense, scale=scale,
                                         kv_heads=kv_heads, seqs=seqs)
        for name, ref in (("dq", dq), ("dk", dk), ("dv", dv)):
            got = to64(gpu[name])
            s = ~np.isnan(ref)
            assert np.all(np.isfinite(got))
            m[name + "_rel_l2"] = rel_l2(got[s], ref[s])
            per_pass, worst = per_pass_rel_l2(got, ref)
            m[name + "_rel_l2_per_pass"] = per_pass
            m[name + "_worst_pass_head"] = worst
    return m


def assert_within(m):
    assert m["o_max_abs"] <= O_MAX_ABS, m
    assert m["lse_max_abs"] <= LSE_MAX_ABS, m
    for k in ("dq_rel_l2", "dk_rel_l2", "dv_rel_l2"):
        if k in m:
            assert m[k] <= GRAD_REL_L2, m
        for e in m.get(k + "_per_pass", []):
            assert e is None or e <= GRAD_REL_L2, (k, m)
