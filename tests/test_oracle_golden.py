"""The oracle on the Tiny workload against its stored regression fixture."""

import os

import numpy as np

from oracle import gsa_oracle as O
from synthetic import generate

PATH = os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.txt")


def _load():
    sel, out, dense = {}, {}, {}
    for line in open(PATH):
        if line.startswith("#"):
            continue
        kind, a, h, *vals = line.split()
        key = (int(a), int(h))
        if kind == "sel":
            sel[key] = [int(v) for v in vals]
        elif kind == "out":
            out[key] = np.array([float(v) for v in vals])
        else:
            dense[key] = np.array([float(v) for v in vals])
    return sel, out, dense


def test_tiny_fixture():
    sel, out, dense = _load()
    x = generate("tiny")
    geo = O.geometry_of(x.workload)
    res = O.gsa_layer(geo, x.q, x.k, x.v, x.w)
    for (a, h), ids in sel.items():
        assert list(res["sel"][a, h]) == ids
    rows = sorted({t for t, _ in out})
    d = O.dense_attention(geo, x.q, x.k, x.v, rows=np.array(rows))
    for (t, h), vals in out.items():
        np.testing.assert_allclose(res["out"][t, h], vals, rtol=0, atol=1e-12)
        np.testing.assert_allclose(d[rows.index(t), h], dense[(t, h)], rtol=0, atol=1e-12)
