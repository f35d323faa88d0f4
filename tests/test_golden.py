"""Hand-derived worked examples stored under tests/golden/ (each file gives
its derivation and the passage it follows), checked against the oracle and,
for the byte sizes, against the library's host-side sizing call."""
import os

import numpy as np

from kv_cache_compression_kv2d_b200 import binding as B

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rows(name):
    out = []
    with open(os.path.join(HERE, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                out.append(line)
    return out


def _fields(name):
    return {k.strip(): v.split() for k, v in (ln.split(":", 1) for ln in _rows(name))}


def test_segment_bytes_golden(orc):
    for ln in _rows("segment_bytes.txt"):
        d, S, r, c, *want = (int(x) for x in ln.split())
        po = orc.params(d, 4, S, 16, r, c, 0.2)
        assert [orc.segment_bytes(po, k) for k in range(4)] == want
        p = B.params(d, 4, 1, S, 16, r, c, 0.2, float(np.float32(d ** -0.5)))
        assert [B.kv2d_segment_bytes(p, k) for k in range(4)] == want


def test_segment_errors_golden(orc):
    f = _fields("segment_errors.txt")
    s = np.array([float(x) for x in f["s"]])
    g = np.array([float(x) for x in f["g"]])
    r = int(f["r"][0])
    p = orc.params(8, 1, len(s), 1, r, 1, 0.2)
    tidx = orc.topr(p, s)
    assert [int(x) for x in tidx] == [int(x) for x in f["tidx"]]
    assert [float(x) for x in orc.segment_errors(p, s, g, tidx)] == [float(x) for x in f["E"]]


def test_budget_walk_golden(orc):
    f = _fields("budget_walk.txt")
    p = orc.params(128, 4, 64, 8, 8, 32, float(np.float32(float(f["beta"][0]))))
    E_all = np.array([[float(x) for x in f["E0"]], [float(x) for x in f["E1"]]])
    st, strat, used = orc.budget(p, E_all)
    assert st == 0
    assert [int(x) for x in strat] == [int(x) for x in f["strategies"]]
    assert used == int(f["used"][0])
