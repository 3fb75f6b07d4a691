"""Write the oracle's regression fixture for the Tiny workload.

Calls only the CPU oracle and the seeded generators.  The values are the
oracle's own (the pages print no worked example); they guard the oracle
against silent drift, while its correctness rests on the pins in
``tests/pins.py``.

    python tests/golden/make_golden.py   # rewrites tests/golden/tiny_oracle.txt
"""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from oracle import gsa_oracle as O  # noqa: E402
from synthetic import generate  # noqa: E402

ROWS = [0, 1, 17, 255, 256, 300, 511]


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


if __name__ == "__main__":
    main()
