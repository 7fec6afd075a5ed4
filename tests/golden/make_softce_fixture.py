"""Writes softce_fixture.txt: the fp64 soft cross-entropy oracle's forward (row losses,
logsumexps, per-pass losses) and backward (dh, dW) of one tiny, fully specified input,
in the pass form and in the general (per-group) form.  Calls the oracle only; rerun it
(from the repository root) only when a change to the oracle's arithmetic is intended and
justified by the pages.

Input: P = 2 passes over two sequences of 3 and 2 tokens (T = 5), hidden size d = 3,
vocabulary V = 4; entries are small rationals chosen by formula (no random generator);
teacher position 3 is masked; pass weights (1, 0.5); upstream gradient 1.5.  The general
form takes 6 rows with explicit teacher positions (one past the teacher rows) in 2
groups."""

import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
from oracle import softce_oracle as sco  # noqa: E402

P, T, D, V = 2, 5, 3, 4
CU = [0, 3, 5]
MASK = np.array([1, 1, 1, 0, 1], dtype=bool)
WEIGHTS = [1.0, 0.5]
GRAD = 1.5
TEACHER = np.array([0, 2, 4, 5, 1, 3])
GROUP = np.array([0, 1, 0, 1, 1, 0])


def inputs():
    i = np.indices((P, T, D)).astype(np.float64)
    h = ((i[0] + 2 * i[1] + 3 * i[2]) % 5 - 2) / 2
    i = np.indices((V, D)).astype(np.float64)
    W = ((2 * i[0] + i[1]) % 7 - 3) / 3
    i = np.indices((T, V)).astype(np.float64)
    y = ((3 * i[0] + 2 * i[1]) % 5 - 2) * 0.75
    return h, W, y


def compute():
    h, W, y = inputs()
    fwd = sco.forward(h, W, y, CU, MASK, WEIGHTS)
    dh, dW = sco.backward(h, W, y, CU, MASK, WEIGHTS, grad=GRAD)
    hg = h.reshape(P * T, D)[:6]
    gen = sco.forward_mapped(hg, W, y, TEACHER, GROUP, 2, MASK, WEIGHTS)
    gdh, gdW = sco.backward_mapped(hg, W, y, TEACHER, GROUP, 2, MASK, WEIGHTS, grad=GRAD)
    return {"rows": fwd["rows"], "lse_z": fwd["lse_z"], "pass_loss": fwd["pass_loss"], "dh": dh, "dW": dW,
            "g_rows": gen["rows"], "g_loss": gen["group_loss"], "g_dh": gdh, "g_dW": gdW}


def write(path):
    with open(path, "w") as f:
        f.write("# fp64 soft-CE oracle on the input defined in make_softce_fixture.py (written by that script)\n")
        for name, a in compute().items():
            a = np.asarray(a)
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
    write(os.path.join(HERE, "softce_fixture.txt"))
