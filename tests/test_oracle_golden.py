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


NEXT_PATH = os.path.join(os.path.dirname(__file__), "golden", "next_rows_oracle.txt")


def test_next_rows_fixture():
    import sys
    sys.path.insert(0, os.path.join(os.path.dirname(__file__), "golden"))
    import make_golden as MG
    vals, sels = {}, {}
    for line in open(NEXT_PATH):
        if line.startswith("#"):
            continue
        kind, a, h, *rest = line.split()
        if kind == "refsel":
            sels[(int(a), int(h))] = [int(v) for v in rest]
        else:
            vals[(kind, int(a), int(h))] = np.array([float(v) for v in rest])
    x = generate(MG.NEXT)
    geo = O.geometry_of(MG.NEXT)
    rows = np.array(MG.NEXT_ROWS)
    got = {"frame": O.frame_attention(geo, x.q, x.k, x.v, rows=rows)}
    for sh, sw in MG.SGA_WINDOWS:
        got[f"sga{sh}x{sw}"] = O.sga_attention(geo, x.q, x.k, x.v, sh, sw, rows=rows)
    ref = O.gsa_layer(O.geometry_of(MG.NEXT.with_(keep=1)), x.q, x.k, x.v, x.w, rows=rows)
    got["refkeep"] = ref["out"]
    for (kind, t, h), want in vals.items():
        np.testing.assert_allclose(got[kind][MG.NEXT_ROWS.index(t), h], want, rtol=0, atol=1e-12)
    for j, a in enumerate(ref["entries"]):
        for h in range(geo.H):
            assert list(ref["sel"][j, h]) == sels[(int(a), h)]
