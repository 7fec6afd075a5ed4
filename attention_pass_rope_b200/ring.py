"""Context-parallel zigzag ring over the pass-1 trunk K/V: the host side.

"DFlash/DSpark and EAGLE-3 TTT draft co-training ..." (NeMo-RL issue 3698), "What I'm
working on", item 4: the pass-1 trunk K/V travels around a ring of ranks and the
partial attentions are joined by the exact log-sum-exp merge.

A sequence of L tokens is cut into 2N chunks for N ranks; rank r holds chunks r and
2N-1-r (the zigzag pairing balances the causal work: an early chunk, little work, with
a late one, much work).  Every rank rotates its own chunks (all passes, at their global
positions) and, for N steps, computes the attention of its query chunks against the
trunk chunks it currently holds -- its own first, then those passed along the ring --
skipping chunks that start after a query chunk (no visible key), merging each partial
into a running result; its own chunk's step also takes the branch keys.  Between steps
the held trunk chunks (rotated pass-1 keys and pass-1 values) go to rank r+1 and come
from rank r-1.  The exchange lands in this GPU's own memory before a kernel reads it.

`ring_forward` is the driver, generic in its step/merge/finish functions and its
exchange; `gpu_ops` returns the CUDA implementations (the C ABI's ttt_ring_* calls)
and `P2PExchange` the torch.distributed one, whose waits are bounded: a rank that
never sends, or sends late, makes its successor raise `RingTimeout` instead of waiting
for ever.
"""

from __future__ import annotations

import ctypes
import dataclasses
import datetime
from typing import Callable, List, Optional, Sequence

import torch

from . import _lib


def zigzag_chunks(L: int, world: int) -> List[tuple]:
    """(start, length) of the 2*world chunks of a sequence of L tokens, as equal as
    possible (the first L % (2*world) chunks one token longer)."""
    n = 2 * world
    base, extra = divmod(L, n)
    out, s = [], 0
    for c in range(n):
        ln = base + (1 if c < extra else 0)
        out.append((s, ln))
        s += ln
    return out


def rank_chunks(rank: int, world: int) -> tuple:
    """Chunk indices held by `rank`: its early and its late chunk."""
    return (rank, 2 * world - 1 - rank)


def ring_schedule(rank: int, world: int) -> List[int]:
    """Rank whose trunk chunks `rank` holds at each step (its own first)."""
    return [(rank - s) % world for s in range(world)]


class RingTimeout(RuntimeError):
    """A peer of the ring did not deliver its chunks within the exchange's time limit."""


@dataclasses.dataclass
class TrunkChunk:
    start: int                 # global position of its first token
    kr: torch.Tensor           # rotated pass-1 keys [Hkv, len, D]
    v: torch.Tensor            # pass-1 values [len, Hkv, D]
    # backward only: the chunk's dk~ / dV accumulators [Hkv, len, D], which travel with it
    dk_acc: Optional[torch.Tensor] = None
    dv_acc: Optional[torch.Tensor] = None


class P2PExchange:
    """Moves the held trunk chunks one rank along the ring with torch.distributed
    send/recv (NCCL between GPUs, gloo on the CPU).  Every wait is bounded by
    `timeout_s`; on expiry it raises RingTimeout.  Receive buffers are allocated on the
    receiver (this rank's memory)."""

    def __init__(self, rank: int, world: int, timeout_s: float = 30.0, group=None):
        self.rank, self.world, self.timeout_s, self.group = rank, world, timeout_s, group

    def _wait(self, works):
        deadline = datetime.timedelta(seconds=self.timeout_s)
        for w in works:
            try:
                ok = w.wait(deadline)
            except RuntimeError as e:  # the backend reports an expired wait as an error
                raise RingTimeout(f"rank {self.rank}: ring exchange did not complete in {self.timeout_s} s") from e
            if ok is False:
                raise RingTimeout(f"rank {self.rank}: ring exchange did not complete in {self.timeout_s} s")

    def shift(self, chunks: Sequence[TrunkChunk], recv_like: Sequence[TrunkChunk]) -> List[TrunkChunk]:
        """Send `chunks` to the next rank, receive as many from the previous one: first
        each chunk's start and length (chunks of a ragged split differ by a token), then
        the keys and values into buffers of the received sizes."""
        dist = torch.distributed
        nxt, prv = (self.rank + 1) % self.world, (self.rank - 1) % self.world
        dev = chunks[0].kr.device
        meta_out = torch.tensor([[c.start, c.kr.shape[1]] for c in chunks], dtype=torch.int64, device=dev)
        meta_in = torch.empty_like(meta_out)
        self._wait(dist.batch_isend_irecv([dist.P2POp(dist.isend, meta_out, nxt, self.group),
                                           dist.P2POp(dist.irecv, meta_in, prv, self.group)]))
        out, ops = [], []
        for c, (start, n), like in zip(chunks, meta_in.tolist(), recv_like):
            r = TrunkChunk(int(start), like.kr.new_empty((like.kr.shape[0], int(n), like.kr.shape[2])),
                           like.v.new_empty((int(n), *like.v.shape[1:])))
            pairs = [(c.kr, r.kr), (c.v, r.v)]
            if c.dk_acc is not None:
                r.dk_acc = c.dk_acc.new_empty((c.dk_acc.shape[0], int(n), c.dk_acc.shape[2]))
                r.dv_acc = c.dv_acc.new_empty((c.dv_acc.shape[0], int(n), c.dv_acc.shape[2]))
                pairs += [(c.dk_acc, r.dk_acc), (c.dv_acc, r.dv_acc)]
            out.append(r)
            for snd, rcv in pairs:
                ops += [dist.P2POp(dist.isend, snd, nxt, self.group), dist.P2POp(dist.irecv, rcv, prv, self.group)]
        self._wait(dist.batch_isend_irecv(ops))
        return out


def ring_forward(local: Sequence[dict], step: Callable, merge: Callable, finish: Callable,
                 exchange, world: int, trunk: Sequence[TrunkChunk]):
    """Run the ring on one rank.

    local: this rank's query chunks, each a dict with at least "start" (global position)
      and whatever `step` needs; trunk: its own trunk chunks (same order).
    step(q_chunk, trunk_chunk, include_branch) -> partial; merge(acc, partial) -> acc
      (acc None on the first call); finish(q_chunk, acc) -> result.
    exchange.shift(held, like) -> the chunks of the previous rank (None for world 1).
    Returns [finish(...) for every local chunk]."""
    acc: List[Optional[object]] = [None] * len(local)
    held = list(trunk)
    for s in range(world):
        if s > 0:
            held = exchange.shift(held, trunk)
        for i, qc in enumerate(local):
            for tc in held:
                if tc.start > qc["start"]:
                    continue  # a chunk that starts later holds no key this chunk sees
                part = step(qc, tc, include_branch=(tc.start == qc["start"]))
                acc[i] = merge(acc[i], part)
    return [finish(qc, a) for qc, a in zip(local, acc)]


def ring_backward(local: Sequence[dict], prepare: Callable, step: Callable, finish: Callable,
                  finish_trunk: Callable, exchange, world: int, trunk: Sequence[TrunkChunk], zeros: Callable):
    """The ring's backward on one rank, after ring_forward.

    local: this rank's query chunks (with whatever the functions need: the final o and
      lse, dout); trunk: its own trunk chunks.
    prepare(q_chunk): delta and the chunk's zeroed dq~ accumulator.
    step(q_chunk, trunk_chunk, include_branch): the pair's contribution -- dq~ into the
      query chunk's accumulator, dk~ / dV into the trunk chunk's travelling accumulators.
    finish(q_chunk) -> the query chunk's dq and branch-pass dK / dV.
    finish_trunk(trunk_chunk) -> its pass-1 dK / dV from its accumulators, home again.
    zeros(trunk_chunk) -> (dk_acc, dv_acc) zeroed.
    The trunk chunks travel as in the forward, each with its accumulators; after the
    ring one more shift brings every accumulator back to its owner.
    Returns ([finish(q) for q in local], [finish_trunk(t) for t in this rank's own])."""
    for qc in local:
        prepare(qc)
    held = []
    for tc in trunk:
        dk_acc, dv_acc = zeros(tc)
        held.append(dataclasses.replace(tc, dk_acc=dk_acc, dv_acc=dv_acc))
    for s in range(world):
        if s > 0:
            held = exchange.shift(held, trunk)
        for qc in local:
            for tc in held:
                if tc.start > qc["start"]:
                    continue  # a chunk that starts later holds no key this chunk sees
                step(qc, tc, include_branch=(tc.start == qc["start"]))
    if world > 1:
        held = exchange.shift(held, trunk)  # the accumulators come home
    return [finish(qc) for qc in local], [finish_trunk(tc) for tc in held]


# ----------------------------------------------------------------------------- CUDA implementation

def _desc(P, H, Hkv, D, theta, scale, q_len, q_start, kv_len=0, kv_start=0, include_branch=False):
    d = _lib.TTTRingDesc()
    d.P, d.H, d.Hkv, d.D = P, H, Hkv, D
    d.rope_theta = float(theta)
    d.softmax_scale = 0.0 if scale is None else float(scale)
    d.q_len, d.q_start, d.kv_len, d.kv_start = q_len, q_start, kv_len, kv_start
    d.include_branch = int(include_branch)
    return d


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _s():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def rotate_chunk(q, k, v, start: int, theta: float, scale=None) -> dict:
    """A local chunk (q [P, len, H, D], k, v [P, len, Hkv, D], bf16, contiguous) with
    its rotated copies; returns the query-chunk dict `ring_forward` takes."""
    P, n, H, D = q.shape
    Hkv = k.shape[2]
    qr = torch.empty(P, H, n, D, dtype=q.dtype, device=q.device)
    kr = torch.empty(P, Hkv, n, D, dtype=k.dtype, device=k.device)
    d = _desc(P, H, Hkv, D, theta, scale, n, start)
    _lib.check(_lib.lib().ttt_ring_rotate(ctypes.byref(d), _p(q), _p(k), _p(qr), _p(kr), _s()), "ttt_ring_rotate")
    return {"start": start, "len": n, "qr": qr, "kr": kr, "v": v, "P": P, "H": H, "Hkv": Hkv, "D": D,
            "theta": theta, "scale": scale}


def trunk_of(chunk: dict) -> TrunkChunk:
    """The chunk's pass-1 trunk keys/values, as they travel around the ring."""
    return TrunkChunk(chunk["start"], chunk["kr"][0].contiguous(), chunk["v"][0].contiguous())


def gpu_ops():
    """(step, merge, finish) on the GPU through the C ABI."""
    status = {}

    def step(qc, tc: TrunkChunk, include_branch: bool):
        P, n, H, D = qc["P"], qc["len"], qc["H"], qc["D"]
        dev = qc["qr"].device
        o = torch.empty(P, n, H, D, dtype=torch.float32, device=dev)
        lse = torch.empty(P, H, n, dtype=torch.float32, device=dev)
        st = status.setdefault(dev, torch.zeros(64, dtype=torch.int32, device=dev))
        d = _desc(P, H, qc["Hkv"], D, qc["theta"], qc["scale"], n, qc["start"], tc.kr.shape[1], tc.start,
                  include_branch)
        _lib.check(_lib.lib().ttt_ring_step(ctypes.byref(d), _p(qc["qr"]), _p(qc["kr"]), _p(qc["v"]), _p(tc.kr),
                                            _p(tc.v), _p(o), _p(lse), _p(st), _s()), "ttt_ring_step")
        return (qc, o, lse)

    def merge(acc, part):
        qc, o, lse = part
        d = _desc(qc["P"], qc["H"], qc["Hkv"], qc["D"], qc["theta"], qc["scale"], qc["len"], qc["start"])
        if acc is None:
            return (qc, o, lse)  # the first partial is the running result
        _, oa, la = acc
        _lib.check(_lib.lib().ttt_ring_merge(ctypes.byref(d), _p(oa), _p(la), _p(o), _p(lse), 0, _s()),
                   "ttt_ring_merge")
        return acc

    def finish(qc, acc):
        _, oa, la = acc
        d = _desc(qc["P"], qc["H"], qc["Hkv"], qc["D"], qc["theta"], qc["scale"], qc["len"], qc["start"])
        o = torch.empty(oa.shape, dtype=torch.bfloat16, device=oa.device)
        _lib.check(_lib.lib().ttt_ring_finish(ctypes.byref(d), _p(oa), _p(o), _s()), "ttt_ring_finish")
        return o, la

    return step, merge, finish


def gpu_bwd_ops(theta: float, scale=None):
    """(prepare, step, finish, finish_trunk, zeros) of the ring's backward on the GPU
    through the C ABI (theta, scale as in the forward).  A query chunk dict needs, besides what rotate_chunk gives, "o" and
    "lse" (the forward's final result) and "do"; prepare adds its workspace."""
    L = _lib.lib()

    def desc_of(qc, tc=None):
        return _desc(qc["P"], qc["H"], qc["Hkv"], qc["D"], qc["theta"], qc["scale"], qc["len"], qc["start"],
                     0 if tc is None else tc.kr.shape[1], 0 if tc is None else tc.start)

    def prepare(qc):
        d = desc_of(qc)
        ws = torch.empty(L.ttt_ring_bwd_workspace_size(ctypes.byref(d)), dtype=torch.uint8, device=qc["qr"].device)
        qc["bwd_ws"] = ws
        _lib.check(L.ttt_ring_bwd_prepare(ctypes.byref(d), _p(qc["o"]), _p(qc["lse"]), _p(qc["do"]), _p(ws),
                                          ws.numel(), _s()), "ttt_ring_bwd_prepare")

    def step(qc, tc: TrunkChunk, include_branch: bool):
        d = desc_of(qc, tc)
        ws = qc["bwd_ws"]
        _lib.check(L.ttt_ring_bwd_step(ctypes.byref(d), _p(qc["qr"]), _p(qc["do"]), _p(tc.kr), _p(tc.v),
                                       _p(tc.dk_acc), _p(tc.dv_acc), _p(ws), ws.numel(), _s()), "ttt_ring_bwd_step")

    def finish(qc):
        d = desc_of(qc)
        ws = qc["bwd_ws"]
        dq = torch.empty_like(qc["do"])
        dk = torch.zeros(qc["P"], qc["len"], qc["Hkv"], qc["D"], dtype=torch.bfloat16, device=dq.device)
        dv = torch.zeros_like(dk)
        _lib.check(L.ttt_ring_bwd_finish(ctypes.byref(d), _p(qc["qr"]), _p(qc["kr"]), _p(qc["v"]), _p(qc["do"]),
                                         _p(qc["lse"]), _p(dq), _p(dk), _p(dv), _p(ws), ws.numel(), _s()),
                   "ttt_ring_bwd_finish")
        return dq, dk, dv

    def finish_trunk(tc: TrunkChunk):
        n, Hkv, D = tc.kr.shape[1], tc.kr.shape[0], tc.kr.shape[2]
        d = _desc(1, Hkv, Hkv, D, theta, scale, n, tc.start)
        dk = torch.empty(n, Hkv, D, dtype=torch.bfloat16, device=tc.kr.device)
        dv = torch.empty_like(dk)
        _lib.check(L.ttt_ring_dkv_finish(ctypes.byref(d), _p(tc.dk_acc), _p(tc.dv_acc), _p(dk), _p(dv), _s()),
                   "ttt_ring_dkv_finish")
        return tc.start, dk, dv

    def zeros(tc: TrunkChunk):
        z = torch.zeros(tc.kr.shape, dtype=torch.float32, device=tc.kr.device)
        return z, torch.zeros_like(z)

    return prepare, step, finish, finish_trunk, zeros
