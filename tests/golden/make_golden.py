"""Writes the fixtures of this folder.

* ``hand_example.json``: a 2-row, 3-word example worked by hand from the definition of the
  loss (the pages print no numeric example). H = I_2 and W = [[0,1],[1,1],[2,1]] give the
  logits z = [[0,1,2],[1,1,1]]; labels [2, 0]. Closed forms, with s = 1 + e + e^2:
  lse = (ln s, 1 + ln 3); loss = (ln s - 2, ln 3); mean = (loss_0 + loss_1) / 2;
  P_0 = (1, e, e^2) / s, P_1 = (1/3, 1/3, 1/3); G_i = (P_i - e_{y_i}) / 2;
  dH_i = sum_v G_iv W_v = (sum_v v G_iv, 0); dW_v = (G_0v, G_1v) because H = I.
  Computed below with ``math`` only: no oracle call.
* ``tiny_oracle_summary.json``: a summary of the oracle's result on the seeded 64 x 256 x
  2048 workload, written by calling only ``oracle/`` and ``workloads/``; it detects any
  later drift of the oracle's arithmetic.

Run from the repository root: ``python tests/golden/make_golden.py``.
"""
import json
import math
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))


def hand_example():
    e = math.e
    s = 1 + e + e * e
    lse = [math.log(s), 1 + math.log(3)]
    loss = [math.log(s) - 2, math.log(3)]
    P = [[1 / s, e / s, e * e / s], [1 / 3, 1 / 3, 1 / 3]]
    y = [2, 0]
    G = [[0.5 * (P[i][v] - (1.0 if v == y[i] else 0.0)) for v in range(3)] for i in range(2)]
    dH = [[sum(v * G[i][v] for v in range(3)), 0.0] for i in range(2)]
    dW = [[G[0][v], G[1][v]] for v in range(3)]
    return dict(source="worked by hand from the definition; the pages print no example",
                H=[[1.0, 0.0], [0.0, 1.0]], W=[[0.0, 1.0], [1.0, 1.0], [2.0, 1.0]],
                labels=y, lse=lse, loss_rows=loss, loss_mean=(loss[0] + loss[1]) / 2,
                dH=dH, dW=dW)


def tiny_summary():
    import numpy as np
    from oracle import lmh_oracle as O
    from workloads import WORKLOADS, make_inputs
    x = make_inputs(WORKLOADS["tiny"])
    f = O.ce_fused(x["H"], x["W"], x["labels"])
    return dict(source="oracle.ce_fused on workloads.WORKLOADS['tiny'] (seed 1234)",
                loss_rows=f["loss_rows"].tolist(), lse=f["lse"].tolist(),
                n_valid=f["n_valid"], dH_norm=float(np.linalg.norm(f["dH"])),
                dW_norm=float(np.linalg.norm(f["dW"])), dW_corner=f["dW"][:4, :4].tolist())


if __name__ == "__main__":
    with open(os.path.join(HERE, "hand_example.json"), "w") as fh:
        json.dump(hand_example(), fh, indent=1)
    with open(os.path.join(HERE, "tiny_oracle_summary.json"), "w") as fh:
        json.dump(tiny_summary(), fh, indent=1)
    print("wrote fixtures")
