"""Write the tiny Complex-KDA golden fixture from the CPU oracle.

Calls only ``oracle`` (and the seeded ``workloads`` generator for the inputs).
The fixture pins the generator (a SHA-256 of the drawn inputs) and the oracle's
float64 outputs for that case, so an accidental change to either is caught:
  python tests/golden/make_golden.py
"""
import hashlib
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from workloads import tiny_ckda  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_ckda_seed0.txt")


def input_digest(inp) -> str:
    h = hashlib.sha256()
    for t in inp.tensors():
        h.update(t.contiguous().view(-1).numpy().tobytes())
    return h.hexdigest()


def main():
    inp = tiny_ckda(0)
    o, sf = oracle.recurrence(inp)
    lines = [
        "# Tiny Complex-KDA case (B=1, H=2, T=64, d_k=d_v=16, fp32, alpha~U[-1,1], beta~U[0,2], S0=0, seed 0)",
        "# written by tests/golden/make_golden.py from the float64 CPU oracle",
        f"inputs_sha256 {input_digest(inp)}",
        f"o_sum {float(o.sum())!r}",
        f"o_abs_sum {float(np.abs(o).sum())!r}",
        f"o_sq_sum {float((o ** 2).sum())!r}",
    ]
    for t in (0, 1, 15, 16, 17, 63):
        for h in range(2):
            lines.append(f"o t={t} h={h} " + " ".join(repr(float(x)) for x in o[0, t, h]))
    for h in range(2):
        for i in range(16):
            lines.append(f"S h={h} row={i} " + " ".join(repr(float(x)) for x in sf[0, h, i]))
    with open(OUT, "w") as f:
        f.write("\n".join(lines) + "\n")
    print("wrote", OUT)


if __name__ == "__main__":
    main()
