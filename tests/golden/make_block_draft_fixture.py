"""Writes block_draft_fixture.txt: the fp64 block-draft oracle's forward (O, lse) and
backward (dqb, dk_ctx, dv_ctx, dkb, dvb) of one tiny, fully specified input.  Calls the
oracle only; rerun it (from the repository root) only when a change to the oracle's
arithmetic is intended and justified by the pages.

Input: a context of L = 6 positions, anchors 0, 2 and 5, blocks of Bs = 3 tokens,
H = 2 query heads, Hkv = 1 KV head, D = 4, theta = 10; entries are small rationals
chosen by formula (no random generator), the softmax scale is 1/sqrt(D)."""

import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
from oracle import block_draft_oracle as bd  # noqa: E402

L, ANCHORS, BS, H, HKV, D, THETA = 6, [0, 2, 5], 3, 2, 1, 4, 10.0


def inputs():
    nb = len(ANCHORS)
    i = np.indices((L, HKV, D)).astype(np.float64)
    k_ctx = ((2 * i[0] + 3 * i[2]) % 7 - 3) / 3
    v_ctx = ((i[0] + 2 * i[2]) % 5 - 2) / 2
    i = np.indices((nb, BS, H, D)).astype(np.float64)
    qb = ((i[0] + 2 * i[1] + 3 * i[2] + i[3]) % 6 - 2.5) / 4
    do = ((3 * i[0] + i[1] + i[2] + 2 * i[3]) % 5 - 2) / 5
    i = np.indices((nb, BS, HKV, D)).astype(np.float64)
    kb = ((2 * i[0] + i[1] + 3 * i[3]) % 5 - 2) / 3
    vb = ((i[0] + 3 * i[1] + i[3]) % 7 - 3) / 4
    return dict(k_ctx=k_ctx, v_ctx=v_ctx, anchors=ANCHORS, qb=qb, kb=kb, vb=vb), do


def compute():
    c, do = inputs()
    O, lse = bd.forward_bruteforce(theta=THETA, **c)
    dqb, dk_ctx, dv_ctx, dkb, dvb = bd.backward_bruteforce(theta=THETA, do=do, **c)
    return {"O": O, "lse": lse, "dqb": dqb, "dk_ctx": dk_ctx, "dv_ctx": dv_ctx, "dkb": dkb, "dvb": dvb}


def write(path):
    with open(path, "w") as f:
        f.write("# fp64 block-draft oracle on the input defined in make_block_draft_fixture.py (written by that script)\n")
        for name, a in compute().items():
            f.write(f"{name} {' '.join(str(x) for x in a.shape)}\n")
            f.write(" ".join(repr(float(x)) for x in a.ravel()) + "\n")


def read(path):
    out = {}
    with open(path) as f:
        lines = [ln for ln in f.read().splitlines() if not ln.startswith("#")]
    for head, body in zip(lines[0::2], lines[1::2]):
        name, *shape = head.split()
        out[name] = np.array([float(x) for x in body.split()]).reshape([int(s) for s in shape])
    return out


if __name__ == "__main__":
    write(os.path.join(HERE, "block_draft_fixture.txt"))
