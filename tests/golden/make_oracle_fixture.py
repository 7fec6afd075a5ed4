"""Writes oracle_fixture_p3.txt: the fp64 oracle's forward (O, lse) and backward (dq, dk,
dv) of one tiny, fully specified input.  Calls the oracle only; rerun it (from the
repository root) only when a change to the oracle's arithmetic is intended and
justified by the pages.

Input: P = 3 passes, L = 4 positions, H = 2 query heads, Hkv = 1 KV head, D = 4,
theta = 10; entries are small rationals chosen by formula (no random generator), the
softmax scale is 1/sqrt(D), RoPE output not rounded (rope_round=None)."""

import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
from oracle import ttt_oracle as orc  # noqa: E402

P, L, H, Hkv, D, THETA = 3, 4, 2, 1, 4, 10.0


def inputs():
    idx = np.indices((P, L, H, D)).astype(np.float64)
    q = ((idx[0] + 2 * idx[1] + 3 * idx[2] + 5 * idx[3]) % 7 - 3) / 4
    idx = np.indices((P, L, Hkv, D)).astype(np.float64)
    k = ((3 * idx[0] + idx[1] + 2 * idx[3]) % 5 - 2) / 2
    v = ((idx[0] + 3 * idx[1] + idx[3]) % 6 - 2.5) / 3
    idx = np.indices((P, L, H, D)).astype(np.float64)
    do = ((2 * idx[0] + idx[1] + idx[2] + 3 * idx[3]) % 5 - 2) / 5
    return q, k, v, do


def compute():
    q, k, v, do = inputs()
    O, lse = orc.forward_bruteforce(q, k, v, THETA, rope_round=None)
    dq, dk, dv = orc.backward_bruteforce(q, k, v, do, THETA, rope_round=None)
    return {"O": O, "lse": lse, "dq": dq, "dk": dk, "dv": dv}


def write(path):
    with open(path, "w") as f:
        f.write("# fp64 oracle on the input defined in make_oracle_fixture.py (written by that script)\n")
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
    write(os.path.join(HERE, "oracle_fixture_p3.txt"))
