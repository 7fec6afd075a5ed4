"""Context-parallel zigzag ring over the pass-1 trunk K/V.

CPU (gloo, world size 2 and 4): the host-side driver moves the trunk chunks around the
ring with torch.distributed and each rank computes its partials from the chunks it
received (the step is the oracle's chunk_partial, so only the exchange and the driver
are under test); the merged results equal the oracle on the whole sequence.  A peer
that never sends makes its successor raise RingTimeout; a late one (inside the limit)
changes nothing.  GPU: the CUDA ring step, merge and finish, with the ranks emulated one
after another on one device, against the oracle."""

import datetime
import os
import socket
import sys
import time

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import ttt_inputs
from attention_pass_rope_b200 import ring
from oracle import ttt_oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_zigzag_chunks_and_schedule():
    for L, W in [(10, 2), (4096, 4), (7, 3), (1, 1)]:
        ch = ring.zigzag_chunks(L, W)
        assert len(ch) == 2 * W and ch[0][0] == 0 and sum(n for _, n in ch) == L
        assert all(a + n == b for (a, n), (b, _) in zip(ch[:-1], ch[1:]))
        assert max(n for _, n in ch) - min(n for _, n in ch) <= 1
        held = sorted(c for r in range(W) for c in ring.rank_chunks(r, W))
        assert held == list(range(2 * W))
        for r in range(W):
            assert sorted(ring.ring_schedule(r, W)) == list(range(W)) and ring.ring_schedule(r, W)[0] == r


def _merge_np(acc, part):
    if acc is None:
        return part
    (oa, la), (ob, lb) = acc, part
    m = np.maximum(la, lb)
    ms = np.where(np.isfinite(m), m, 0.0)
    l = ms + np.log(np.exp(la - ms) + np.exp(lb - ms))
    wa = np.where(np.isfinite(l), np.exp(la - l), 0.0).transpose(0, 2, 1)[..., None]
    wb = np.where(np.isfinite(l), np.exp(lb - l), 0.0).transpose(0, 2, 1)[..., None]
    return wa * oa + wb * ob, l


def _cpu_rank(rank, world, port, out, L, drop_rank, delay_rank, timeout_s, with_bwd=False):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        w = ttt_inputs.thd("ring", [L], 3, 4, 2, 16, 1e4)
        inp = ttt_inputs.make_inputs(w, with_grad=with_bwd)
        q, k, v = (t.double().numpy() for t in (inp.q, inp.k, inp.v))
        chunks = ring.zigzag_chunks(L, world)
        local, trunk = [], []
        for c in ring.rank_chunks(rank, world):
            a, n = chunks[c]
            local.append({"start": a, "q": q[:, a:a + n], "k": k[:, a:a + n], "v": v[:, a:a + n]})
            # what travels: this chunk's pass-1 keys ([Hkv, len, D], unrotated here: the
            # oracle rotates them) and values ([len, Hkv, D])
            trunk.append(ring.TrunkChunk(a, inp.k[0, a:a + n].double().transpose(0, 1).contiguous(),
                                         inp.v[0, a:a + n].double().contiguous()))

        def step(qc, tc, include_branch):
            kt = tc.kr.transpose(0, 1).numpy()
            return orc.chunk_partial(qc["q"], kt, tc.v.numpy(), 1e4, qc["start"], tc.start,
                                     branch_k=qc["k"] if include_branch else None,
                                     branch_v=qc["v"] if include_branch else None)

        class Ex(ring.P2PExchange):
            def shift(self, held, like):
                if rank == drop_rank:
                    time.sleep(timeout_s + 2)  # never posts its send
                    raise RuntimeError("dropped")
                if rank == delay_rank:
                    time.sleep(timeout_s / 4)
                return super().shift(held, like)

        ex = Ex(rank, world, timeout_s)
        res = ring.ring_forward(local, step, _merge_np, lambda qc, acc: acc, ex, world, trunk)
        if not with_bwd:
            out[rank] = ("ok", [(qc["start"], o, l) for qc, (o, l) in zip(local, res)])
            return
        # backward: the forward's final (o, lse) per chunk, dO, the oracle's pair
        # contributions as the step; the trunk chunks' accumulators travel with them
        dO = inp.do.double().numpy()
        for qc, (o, l) in zip(local, res):
            a, n = qc["start"], qc["q"].shape[1]
            qc.update(o=o, lse=l, do=dO[:, a:a + n], delta=np.einsum("plhd,plhd->phl", dO[:, a:a + n], o))

        def prepare(qc):
            qc["dq"] = np.zeros_like(qc["q"])

        def bstep(qc, tc, include_branch):
            r = orc.chunk_backward_partial(qc["q"], tc.kr.transpose(0, 1).numpy(), tc.v.numpy(), qc["do"],
                                           qc["lse"], qc["delta"], 1e4, qc["start"], tc.start,
                                           branch_k=qc["k"] if include_branch else None,
                                           branch_v=qc["v"] if include_branch else None)
            qc["dq"] += r[0]
            tc.dk_acc += torch.from_numpy(r[1].transpose(1, 0, 2).copy())
            tc.dv_acc += torch.from_numpy(r[2].transpose(1, 0, 2).copy())
            if include_branch:
                qc["dkb"], qc["dvb"] = r[3], r[4]

        zeros = lambda tc: (torch.zeros_like(tc.kr), torch.zeros_like(tc.kr))  # both [Hkv, len, D]  # noqa: E731
        grads, trunk_g = ring.ring_backward(local, prepare, bstep,
                                            lambda qc: (qc["start"], qc["dq"], qc["dkb"], qc["dvb"]),
                                            lambda tc: (tc.start, tc.dk_acc.numpy(), tc.dv_acc.numpy()),
                                            ex, world, trunk, zeros)
        out[rank] = ("ok", grads, trunk_g)
    except ring.RingTimeout as e:
        out[rank] = ("timeout", str(e))
    except RuntimeError as e:
        out[rank] = ("error", str(e))
    finally:
        os._exit(0)  # a rank whose peer vanished must not wait in the group's teardown


def _run_ring(world, L=37, drop_rank=-1, delay_rank=-1, timeout_s=4.0, with_bwd=False):
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        ps = [ctx.Process(target=_cpu_rank, args=(r, world, port, out, L, drop_rank, delay_rank, timeout_s, with_bwd))
              for r in range(world)]
        for p in ps:
            p.start()
        for p in ps:
            p.join(120)
            assert p.exitcode == 0
        return dict(out)


@pytest.mark.parametrize("world", [2, 4])
def test_ring_over_gloo_ranks_equals_the_oracle(world):
    L = 37  # chunks of 4 and 5 tokens (ragged)
    res = _run_ring(world, L)
    w = ttt_inputs.thd("ring", [L], 3, 4, 2, 16, 1e4)
    inp = ttt_inputs.make_inputs(w, with_grad=False)
    O, lse = orc.forward_twopart(*(t.double().numpy() for t in (inp.q, inp.k, inp.v)), 1e4)
    seen = 0
    for r in range(world):
        kind, chunks = res[r]
        assert kind == "ok", res[r]
        for a, o, l in chunks:
            n = o.shape[1]
            np.testing.assert_allclose(o, O[:, a:a + n], atol=1e-12)
            np.testing.assert_allclose(l, lse[:, :, a:a + n], atol=1e-12)
            seen += n
    assert seen == L


@pytest.mark.parametrize("world", [2, 4])
def test_ring_backward_over_gloo_ranks_equals_the_oracle(world):
    """The ring's backward: each rank adds its query chunks' contributions (the oracle's
    pair contributions, from the forward's final lse) while the trunk chunks travel with
    their dk / dV accumulators, which one more shift brings home; gathered, dq, dk and
    dv equal the oracle's backward on the whole sequence."""
    L = 37
    res = _run_ring(world, L, with_bwd=True)
    w = ttt_inputs.thd("ring", [L], 3, 4, 2, 16, 1e4)
    inp = ttt_inputs.make_inputs(w)
    q, k, v, do = (t.double().numpy() for t in (inp.q, inp.k, inp.v, inp.do))
    O, lse = orc.forward_twopart(q, k, v, 1e4)
    dq, dk, dv = orc.backward_twopart(q, k, v, do, lse, 1e4)
    gq, gk, gv = np.full_like(dq, np.nan), np.full_like(dk, np.nan), np.full_like(dv, np.nan)
    for r in range(world):
        assert res[r][0] == "ok", res[r]
        for a, dqc, dkb, dvb in res[r][1]:
            n = dqc.shape[1]
            gq[:, a:a + n] = dqc
            gk[1:, a:a + n] = dkb[1:]
            gv[1:, a:a + n] = dvb[1:]
        for a, dka, dva in res[r][2]:
            n = dva.shape[1]
            gk[0, a:a + n] = dka.transpose(1, 0, 2)
            gv[0, a:a + n] = dva.transpose(1, 0, 2)
    np.testing.assert_allclose(gq, dq, atol=1e-11)
    np.testing.assert_allclose(gk, dk, atol=1e-11)
    np.testing.assert_allclose(gv, dv, atol=1e-11)


def test_ring_late_peer_inside_the_limit():
    res = _run_ring(2, delay_rank=1, timeout_s=4.0)
    assert all(res[r][0] == "ok" for r in range(2)), res


def test_ring_dropped_peer_raises_timeout():
    """Rank 1 never sends: rank 0's bounded wait ends with RingTimeout (no hang)."""
    t0 = time.time()
    res = _run_ring(2, drop_rank=1, timeout_s=2.0)
    assert res[0][0] == "timeout", res
    assert time.time() - t0 < 90


# ----------------------------------------------------------------------------- GPU

needs_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


class _EmulatedExchange:
    """All ranks' trunk chunks on one device: step s of rank r holds rank (r - s)'s."""

    def __init__(self, rank, world, trunks):
        self.rank, self.world, self.trunks, self.s = rank, world, trunks, 0

    def shift(self, held, like):
        self.s += 1
        return self.trunks[(self.rank - self.s) % self.world]


@pytest.mark.gpu
@needs_cuda
@pytest.mark.parametrize("world,L,P,H,Hkv,D", [(2, 1000, 3, 8, 2, 128), (4, 4096, 3, 32, 8, 128),
                                               (3, 777, 5, 4, 1, 64),
                                               # chunks shorter than a tile, no branch keys (P = 1),
                                               # a group of 3, four passes over uneven chunks
                                               (2, 129, 2, 2, 1, 64), (4, 333, 1, 6, 2, 128),
                                               (3, 2500, 4, 8, 4, 128)])
def test_ring_cuda_steps_emulated_on_one_device(world, L, P, H, Hkv, D):
    """The zigzag ring's CUDA steps (rotation at global positions, partial attention of a
    query chunk against a visiting trunk chunk, log-sum-exp merge, bf16 finish), all
    ranks emulated one after another on one device, against the oracle on the whole
    sequence: O max-abs <= 2e-2, lse max-abs <= 1e-3."""
    from tests import parity
    w = ttt_inputs.thd("ring_gpu", [L], P, H, Hkv, D, 1e6)
    inp = ttt_inputs.make_inputs(w, with_grad=False)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    chunks = ring.zigzag_chunks(L, world)
    local = {}
    for r in range(world):
        local[r] = []
        for c in ring.rank_chunks(r, world):
            a, n = chunks[c]
            local[r].append(ring.rotate_chunk(q[:, a:a + n].contiguous(), k[:, a:a + n].contiguous(),
                                              v[:, a:a + n].contiguous(), a, w.theta))
    trunks = {r: [ring.trunk_of(c) for c in local[r]] for r in range(world)}
    step, merge, finish = ring.gpu_ops()
    o = torch.full((P, L, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((P, H, L), float("nan"), device="cuda")
    for r in range(world):
        res = ring.ring_forward(local[r], step, merge, finish, _EmulatedExchange(r, world, trunks), world, trunks[r])
        for qc, (oc, lc) in zip(local[r], res):
            a, n = qc["start"], qc["len"]
            o[:, a:a + n] = oc
            lse[:, :, a:a + n] = lc
    torch.cuda.synchronize()
    kv = [Hkv - 1] if H > 8 else None
    m = parity.compare_full(w, inp, {"o": o, "lse": lse}, with_grad=False, kv_heads=kv)
    print("ring", world, L, m)
    parity.assert_within(m)


@pytest.mark.gpu
@needs_cuda
@pytest.mark.parametrize("world,L,P,H,Hkv,D", [(2, 1000, 3, 8, 2, 128), (4, 4096, 3, 32, 8, 128),
                                               (3, 777, 5, 4, 1, 64),
                                               # chunks shorter than a tile, no branch keys (P = 1),
                                               # a group of 3, four passes over uneven chunks
                                               (2, 129, 2, 2, 1, 64), (4, 333, 1, 6, 2, 128),
                                               (3, 2500, 4, 8, 4, 128)])
def test_ring_backward_cuda_emulated_on_one_device(world, L, P, H, Hkv, D):
    """The ring's CUDA backward: every rank's prepare (delta, statistics, zeroed dq~),
    its steps against the trunk chunks it would hold (dq~ into the query chunk's
    accumulator, dk~ / dV into the trunk chunk's fp32 accumulators, which in a real ring
    travel with it and come home), the branch part and dq finish, and the trunk chunks'
    dK / dV finish; the ranks one after another on one device, after the CUDA forward
    ring.  Against the oracle's backward on the whole sequence: dq, dk, dv relative L2 <=
    1e-2 (per pass too)."""
    from tests import parity
    w = ttt_inputs.thd("ring_gpu", [L], P, H, Hkv, D, 1e6)
    inp = ttt_inputs.make_inputs(w)
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.do))
    chunks = ring.zigzag_chunks(L, world)
    local = {}
    for r in range(world):
        local[r] = []
        for c in ring.rank_chunks(r, world):
            a, n = chunks[c]
            qc = ring.rotate_chunk(q[:, a:a + n].contiguous(), k[:, a:a + n].contiguous(), v[:, a:a + n].contiguous(),
                                   a, w.theta)
            qc["do"] = do[:, a:a + n].contiguous()
            local[r].append(qc)
    trunks = {r: [ring.trunk_of(c) for c in local[r]] for r in range(world)}
    step, merge, finish = ring.gpu_ops()
    o = torch.full((P, L, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((P, H, L), float("nan"), device="cuda")
    for r in range(world):
        res = ring.ring_forward(local[r], step, merge, finish, _EmulatedExchange(r, world, trunks), world, trunks[r])
        for qc, (oc, lc) in zip(local[r], res):
            qc["o"], qc["lse"] = oc, lc.contiguous()
            o[:, qc["start"]:qc["start"] + qc["len"]] = oc
            lse[:, :, qc["start"]:qc["start"] + qc["len"]] = lc
    prepare, bstep, bfinish, finish_trunk, zeros = ring.gpu_bwd_ops(w.theta)
    # every trunk chunk's accumulators, shared by the emulated ranks
    for r in range(world):
        trunks[r] = [ring.TrunkChunk(tc.start, tc.kr, tc.v, *zeros(tc)) for tc in trunks[r]]
    for r in range(world):
        for qc in local[r]:
            prepare(qc)
    for r in range(world):
        for s in range(world):
            for qc in local[r]:
                for tc in trunks[(r - s) % world]:
                    if tc.start <= qc["start"]:
                        bstep(qc, tc, tc.start == qc["start"])
    dq = torch.full((P, L, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    dk = torch.full((P, L, Hkv, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    dv = torch.full_like(dk, float("nan"))
    for r in range(world):
        for qc in local[r]:
            a, n = qc["start"], qc["len"]
            dqc, dkc, dvc = bfinish(qc)
            dq[:, a:a + n] = dqc
            dk[1:, a:a + n] = dkc[1:]
            dv[1:, a:a + n] = dvc[1:]
        for tc in trunks[r]:
            a, dkt, dvt = finish_trunk(tc)
            dk[0, a:a + dkt.shape[0]] = dkt
            dv[0, a:a + dvt.shape[0]] = dvt
    torch.cuda.synchronize()
    kv = [Hkv - 1] if H > 8 else None
    m = parity.compare_full(w, inp, {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv}, kv_heads=kv)
    print("ring bwd", world, L, m)
    parity.assert_within(m)
