"""Seeded synthetic inputs for the multi-pass TTT trunk+branch attention, the block-draft
attention and the draft's soft cross-entropy distillation loss.

This module is the only code shared by the fp64 oracle (``oracle/``) and the
CUDA path (``attention_pass_rope_b200``).  It draws random numbers and packs
them into tensors; it holds none of the method's arithmetic (no RoPE, no
softmax, no masking, no teacher alignment).

Recipe (the same for every workload):

* one ``torch.Generator`` on the CPU, seeded with ``seed``;
* for packed variable-length (THD) workloads the sequence lengths are drawn
  first, ``torch.randint(lo, hi + 1, (nseq,))``;
* then, in this order, Q ``[P, T, H, D]``, K ``[P, T, Hkv, D]``,
  V ``[P, T, Hkv, D]`` and the output gradient dO ``[P, T, H, D]``, each
  fp32 N(0, 1) times ``scale`` and rounded to bf16 (round to nearest even,
  torch's cast).

Dense ``[B, S, ...]`` batches are stored pass-major as ``[P, B*S, ...]``: the
token axis of a dense batch is the concatenation of its B sequences, so a
dense batch is the THD layout with ``cu_seqlens = [0, S, 2S, ..., B*S]``.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape of one attention call.

    ``lengths`` lists the sequence lengths; a dense batch has ``B`` equal
    lengths ``S``.  ``dense`` selects the public lse layout ``[P, B, H, S]``
    (dense) or ``[P, H, T]`` (THD).
    """

    name: str
    P: int
    H: int
    Hkv: int
    D: int
    theta: float
    lengths: tuple
    dense: bool
    scale: float = 1.0
    seed: int = 0
    len_range: tuple = ()   # (lo, hi) when the lengths were drawn from the generator

    @property
    def T(self) -> int:
        return int(sum(self.lengths))

    @property
    def nseq(self) -> int:
        return len(self.lengths)

    @property
    def max_seqlen(self) -> int:
        return int(max(self.lengths))

    @property
    def cu_seqlens(self) -> list:
        out = [0]
        for n in self.lengths:
            out.append(out[-1] + int(n))
        return out

    @property
    def trunk_pairs(self) -> int:
        """Visible (query, trunk key) pairs summed over sequences, per head and pass."""
        return int(sum(n * (n + 1) // 2 for n in self.lengths))

    def flops_fwd_bwd(self, per_pair: int = 14) -> float:
        """Algorithmic flops: ``per_pair * D`` per visible trunk pair, head and pass,
        plus the branch keys (4*D fwd + 10*D bwd per branch key and query)."""
        trunk = per_pair * self.D * self.trunk_pairs * self.H * self.P
        branch_keys = self.T * self.H * sum(p - 1 for p in range(1, self.P + 1))
        return float(trunk + per_pair * self.D * branch_keys)

    def flops_fwd(self) -> float:
        return self.flops_fwd_bwd(per_pair=4)


def dense(name, B, S, P, H, Hkv, D, theta, scale=1.0, seed=0) -> Workload:
    return Workload(name, P, H, Hkv, D, float(theta), tuple([S] * B), True, scale, seed)


def thd(name, lengths, P, H, Hkv, D, theta, scale=1.0, seed=0) -> Workload:
    return Workload(name, P, H, Hkv, D, float(theta), tuple(int(x) for x in lengths), False, scale, seed)


def thd_random_lengths(name, nseq, lo, hi, P, H, Hkv, D, theta, scale=1.0, seed=0) -> Workload:
    g = torch.Generator().manual_seed(seed)
    lengths = torch.randint(lo, hi + 1, (nseq,), generator=g).tolist()
    w = thd(name, lengths, P, H, Hkv, D, theta, scale, seed)
    return dataclasses.replace(w, len_range=(lo, hi))


# The five workloads the method is measured on (sizes from the benchmark spec).
def workloads() -> dict:
    return {
        "tiny": dense("tiny", B=1, S=128, P=3, H=4, Hkv=2, D=64, theta=1e4),
        "qwen3_8b_4k": dense("qwen3_8b_4k", B=2, S=4096, P=3, H=32, Hkv=8, D=128, theta=1e6),
        "deep_ttt_8k": dense("deep_ttt_8k", B=1, S=8192, P=7, H=32, Hkv=8, D=128, theta=1e6),
        "thd_packed": thd_random_lengths("thd_packed", nseq=16, lo=256, hi=4096, P=3, H=32, Hkv=8,
                                         D=128, theta=1e6),
        "long_32k": dense("long_32k", B=1, S=32768, P=5, H=32, Hkv=8, D=128, theta=1e6, scale=0.5),
    }


@dataclasses.dataclass
class Inputs:
    """bf16 tensors on the CPU, pass-major, token axis packed."""

    q: torch.Tensor   # [P, T, H, D]
    k: torch.Tensor   # [P, T, Hkv, D]
    v: torch.Tensor   # [P, T, Hkv, D]
    do: torch.Tensor  # [P, T, H, D]


def make_inputs(w: Workload, with_grad: bool = True, seed: Optional[int] = None) -> Inputs:
    """Draw the inputs of ``w`` in the documented order (see module docstring)."""
    g = torch.Generator().manual_seed(w.seed if seed is None else seed)
    if w.len_range and (seed is None or seed == w.seed):
        # the lengths were the first draw of this generator: replay it
        lo, hi = w.len_range
        drawn = torch.randint(lo, hi + 1, (w.nseq,), generator=g).tolist()
        assert tuple(drawn) == w.lengths

    def draw(*shape):
        x = torch.randn(*shape, generator=g, dtype=torch.float32)
        if w.scale != 1.0:
            x.mul_(w.scale)
        return x.to(torch.bfloat16)

    T = w.T
    q = draw(w.P, T, w.H, w.D)
    k = draw(w.P, T, w.Hkv, w.D)
    v = draw(w.P, T, w.Hkv, w.D)
    do = draw(w.P, T, w.H, w.D) if with_grad else None
    return Inputs(q, k, v, do)


# ----------------------------------------------------------------------------- block-draft attention

@dataclasses.dataclass(frozen=True)
class BlockWorkload:
    """Shape of one block-draft call: per sequence a context of ``ctx_lengths[n]`` tokens
    and ``nblocks[n]`` blocks of ``Bs`` tokens.  Anchors are drawn per sequence (sorted
    uniform positions of its context) unless ``anchors`` lists them (flat, per block)."""

    name: str
    H: int
    Hkv: int
    D: int
    Bs: int
    theta: float
    ctx_lengths: tuple
    nblocks: tuple
    dense: bool
    scale: float = 1.0
    seed: int = 0
    anchors: tuple = ()

    @property
    def nseq(self) -> int:
        return len(self.ctx_lengths)

    @property
    def Tc(self) -> int:
        return int(sum(self.ctx_lengths))

    @property
    def NB(self) -> int:
        return int(sum(self.nblocks))

    @property
    def cu_ctx(self) -> list:
        out = [0]
        for n in self.ctx_lengths:
            out.append(out[-1] + int(n))
        return out

    @property
    def cu_blocks(self) -> list:
        out = [0]
        for n in self.nblocks:
            out.append(out[-1] + int(n))
        return out

    def flops_fwd_bwd(self, anchors, per_pair: int = 14) -> float:
        """Algorithmic flops: ``per_pair * D`` per visible (block token, key) pair and query
        head: (anchor + 1) trunk keys and Bs block keys per block token."""
        keys = sum((int(a) + 1 + self.Bs) * self.Bs for a in anchors)
        return float(per_pair * self.D * keys * self.H)


def block_dense(name, B, S, nblk, Bs, H, Hkv, D, theta, scale=1.0, seed=0, anchors=()) -> BlockWorkload:
    return BlockWorkload(name, H, Hkv, D, Bs, float(theta), tuple([S] * B), tuple([nblk] * B), True, scale, seed,
                         tuple(anchors))


def block_thd(name, ctx_lengths, nblocks, Bs, H, Hkv, D, theta, scale=1.0, seed=0, anchors=()) -> BlockWorkload:
    return BlockWorkload(name, H, Hkv, D, Bs, float(theta), tuple(int(x) for x in ctx_lengths),
                         tuple(int(x) for x in nblocks), False, scale, seed, tuple(anchors))


def block_workloads() -> dict:
    """Block-draft workloads with the draft layer's head shapes (32/8 heads, D = 128)."""
    return {
        "block_tiny": block_dense("block_tiny", B=1, S=128, nblk=8, Bs=4, H=4, Hkv=2, D=64, theta=1e4),
        "block_draft_4k": block_dense("block_draft_4k", B=2, S=4096, nblk=256, Bs=16, H=32, Hkv=8, D=128,
                                      theta=1e6),
    }


@dataclasses.dataclass
class BlockInputs:
    """bf16 tensors on the CPU (packed layouts) and int32 anchors (flat, per block)."""

    k_ctx: torch.Tensor   # [Tc, Hkv, D]
    v_ctx: torch.Tensor   # [Tc, Hkv, D]
    qb: torch.Tensor      # [NB, Bs, H, D]
    kb: torch.Tensor      # [NB, Bs, Hkv, D]
    vb: torch.Tensor      # [NB, Bs, Hkv, D]
    do: torch.Tensor      # [NB, Bs, H, D]
    anchors: torch.Tensor  # [NB] int32


def make_block_inputs(w: BlockWorkload) -> BlockInputs:
    """One generator seeded with ``w.seed``: the anchors first (per sequence, sorted
    ``randint(0, L_n)`` draws, unless given), then K_ctx, V_ctx, Qb, Kb, Vb and dO, each
    fp32 N(0, 1) times ``scale`` rounded to bf16."""
    g = torch.Generator().manual_seed(w.seed)
    if w.anchors:
        anchors = torch.tensor(w.anchors, dtype=torch.int32)
        assert anchors.numel() == w.NB
    else:
        parts = [torch.sort(torch.randint(0, max(L, 1), (nb,), generator=g)).values
                 for L, nb in zip(w.ctx_lengths, w.nblocks)]
        anchors = (torch.cat(parts) if parts else torch.zeros(0, dtype=torch.int64)).to(torch.int32)

    def draw(*shape):
        x = torch.randn(*shape, generator=g, dtype=torch.float32)
        if w.scale != 1.0:
            x.mul_(w.scale)
        return x.to(torch.bfloat16)

    k_ctx = draw(w.Tc, w.Hkv, w.D)
    v_ctx = draw(w.Tc, w.Hkv, w.D)
    qb = draw(w.NB, w.Bs, w.H, w.D)
    kb = draw(w.NB, w.Bs, w.Hkv, w.D)
    vb = draw(w.NB, w.Bs, w.Hkv, w.D)
    do = draw(w.NB, w.Bs, w.H, w.D)
    return BlockInputs(k_ctx, v_ctx, qb, kb, vb, do, anchors)


@dataclasses.dataclass(frozen=True)
class SoftCEWorkload:
    """Shape of one distillation-loss call: P draft passes over the tokens of ``lengths``
    (sequences packed back to back), hidden size d, vocabulary V."""

    name: str
    P: int
    lengths: tuple
    d: int
    V: int
    seed: int = 0
    mask_keep: float = 0.9   # probability that a teacher position is counted

    @property
    def T(self) -> int:
        return int(sum(self.lengths))

    @property
    def cu_seqlens(self) -> list:
        out = [0]
        for n in self.lengths:
            out.append(out[-1] + int(n))
        return out

    def flops_fwd(self) -> float:
        """The logits GEMM of every (pass, token) row: 2 * d * V per row."""
        return 2.0 * self.P * self.T * self.d * self.V

    def flops_fwd_bwd(self, with_dw: bool = True) -> float:
        """The algorithmic work of forward and backward: the logits, dh and (optionally) dW,
        2 * d * V each per row (a recomputation of the logits is not counted)."""
        return self.flops_fwd() * (3.0 if with_dw else 2.0)


def softce_workloads() -> dict:
    """Distillation-loss workloads with the Qwen3-8B head (d = 4096, V = 151936)."""
    return {
        "softce_tiny": SoftCEWorkload("softce_tiny", P=3, lengths=(70, 129, 1, 56), d=128, V=1000),
        "softce_mid": SoftCEWorkload("softce_mid", P=3, lengths=(300, 129, 571), d=512, V=8200),
        "softce_qwen3_8b_4k": SoftCEWorkload("softce_qwen3_8b_4k", P=3, lengths=(4096, 4096), d=4096, V=151936),
        # a 32K draft vocabulary (EAGLE-3 drafters may predict a reduced vocabulary): the
        # profiling case of the same kernels, a few GB on the device
        "softce_qwen3_8b_v32k": SoftCEWorkload("softce_qwen3_8b_v32k", P=3, lengths=(2048, 2048), d=4096, V=32768),
    }


@dataclasses.dataclass
class SoftCEInputs:
    """bf16 tensors on the CPU and the uint8 loss mask."""

    h: torch.Tensor      # [P, T, d] draft hidden states
    W: torch.Tensor      # [V, d] vocabulary head
    y: torch.Tensor      # [T, V] teacher logits
    mask: torch.Tensor   # [T] uint8, 1 = teacher position counted


def make_softce_inputs(w: SoftCEWorkload) -> SoftCEInputs:
    """One generator seeded with ``w.seed``, drawn in this order: h (N(0, 1), the scale
    of a normalised hidden state), W (N(0, 1) / sqrt(d), so that a logit has unit scale
    times 2), y (N(0, 1) times 3: a teacher sharper than the draft) and the mask
    (Bernoulli(mask_keep)); the floating tensors are rounded to bf16."""
    g = torch.Generator().manual_seed(w.seed)
    h = torch.randn(w.P, w.T, w.d, generator=g).to(torch.bfloat16)
    W = (torch.randn(w.V, w.d, generator=g) * (2.0 / w.d ** 0.5)).to(torch.bfloat16)
    y = (torch.randn(w.T, w.V, generator=g) * 3.0).to(torch.bfloat16)
    mask = (torch.rand(w.T, generator=g) < w.mask_keep).to(torch.uint8)
    return SoftCEInputs(h, W, y, mask)
