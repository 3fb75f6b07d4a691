"""Write the oracle's regression fixtures: the Tiny workload's GSA layer and
dense attention, and the next rows (frame attention, subsampled global
attention, the reference-frame keep) on a small Gaussian workload.

Calls only the CPU oracle and the seeded generators.  The values are the
oracle's own (the pages print no worked example); they guard the oracle
against silent drift, while its correctness rests on the pins in
``tests/pins.py``.

    python tests/golden/make_golden.py   # rewrites tests/golden/*_oracle.txt
"""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from oracle import gsa_oracle as O  # noqa: E402
from synthetic import Workload, generate  # noqa: E402

ROWS = [0, 1, 17, 255, 256, 300, 511]
# 3 frames x (2 specials + 10 x 11 patches), 2 heads, pool 3, K = 5
NEXT = Workload("next_rows", 3, 2, 10, 11, 2, 64, 3, 5, 21, "gaussian")
NEXT_ROWS = [0, 1, 2, 13, 111, 112, 150, 223, 300, 335]
SGA_WINDOWS = [(2, 2), (3, 2)]


def main(path=os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.txt")):
    x = generate("tiny")
    geo = O.geometry_of(x.workload)
    res = O.gsa_layer(geo, x.q, x.k, x.v, x.w)
    dense = O.dense_attention(geo, x.q, x.k, x.v, rows=np.array(ROWS))
    with open(path, "w") as f:
        f.write("# Tiny workload (N=2, 16x16, S=0, H=2, D=64, P=4, K=4, Gaussian seed 0).\n")
        f.write("# Written by tests/golden/make_golden.py from the CPU oracle only.\n")
        for a in range(res["sel"].shape[0]):
            for h in range(geo.H):
                f.write(f"sel {a} {h} " + " ".join(str(int(b)) for b in res["sel"][a, h]) + "\n")
        for i, t in enumerate(ROWS):
            for h in range(geo.H):
                f.write(f"out {t} {h} " + " ".join(f"{v:.17g}" for v in res["out"][t, h]) + "\n")
                f.write(f"dense {t} {h} " + " ".join(f"{v:.17g}" for v in dense[i, h]) + "\n")


def main_next(path=os.path.join(os.path.dirname(os.path.abspath(__file__)), "next_rows_oracle.txt")):
    x = generate(NEXT)
    geo = O.geometry_of(NEXT)
    rows = np.array(NEXT_ROWS)
    frame = O.frame_attention(geo, x.q, x.k, x.v, rows=rows)
    sga = {w: O.sga_attention(geo, x.q, x.k, x.v, *w, rows=rows) for w in SGA_WINDOWS}
    ref_geo = O.geometry_of(NEXT.with_(keep=1))
    ref = O.gsa_layer(ref_geo, x.q, x.k, x.v, x.w, rows=rows)
    with open(path, "w") as f:
        f.write("# 3 frames x (2 specials + 10x11 patches), H=2, D=64, P=3, K=5, Gaussian seed 21.\n")
        f.write("# Written by tests/golden/make_golden.py from the CPU oracle only.\n")
        for i, t in enumerate(NEXT_ROWS):
            for h in range(geo.H):
                f.write(f"frame {t} {h} " + " ".join(f"{v:.17g}" for v in frame[i, h]) + "\n")
                for (sh, sw), o in sga.items():
                    f.write(f"sga{sh}x{sw} {t} {h} " + " ".join(f"{v:.17g}" for v in o[i, h]) + "\n")
                f.write(f"refkeep {t} {h} " + " ".join(f"{v:.17g}" for v in ref["out"][i, h]) + "\n")
        for j, a in enumerate(ref["entries"]):
            for h in range(geo.H):
                f.write(f"refsel {a} {h} " + " ".join(str(int(b)) for b in ref["sel"][j, h]) + "\n")


if __name__ == "__main__":
    main()
    main_next()
