"""Write tests/golden/oracle_snapshot.txt from the oracle alone.

A regression snapshot, not an independent pin: for the small workloads it
records SHA-256 digests of every integer output of the oracle's quantisation
and selection (codes, block scales, tensor scales' bit patterns, V exponents,
BF16 masks), so that any later change to the oracle's arithmetic shows up as
a failing test and has to be justified by the passage it follows.  Run from
the repository root:  python tests/golden/make_oracle_snapshot.py
"""
import hashlib
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from mixed_precision_bit_quant_b200 import workloads  # noqa: E402  (seeded input generator only)
from oracle import quantize as oq  # noqa: E402
from oracle import select as osel  # noqa: E402

WORKLOADS = ("tiny", "vit")
OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_snapshot.txt")


def digest(a) -> str:
    a = np.ascontiguousarray(np.asarray(a))
    return hashlib.sha256(a.dtype.str.encode() + str(a.shape).encode() + a.tobytes()).hexdigest()


def snapshot_lines():
    lines = []
    for name in WORKLOADS:
        w = workloads.WORKLOADS[name]
        q, k, v = workloads.generate(w)
        quant = oq.quantize(q, k, v)
        for field in ("q_codes", "q_sf", "q_g", "k_codes", "k_sf", "k_g", "v_code", "v_exp"):
            a = np.asarray(quant[field])
            if a.dtype == np.float32:
                a = a.view(np.uint32)  # tensor scales by bit pattern
            lines.append(f"{name} {field} {digest(a)}")
        sel = osel.select(q, k, w.causal, w.budget_bp, w.budget_tiles)
        lines.append(f"{name} mask {digest(sel['mask'])}")
        lines.append(f"{name} counts {digest(sel['counts'])}")
    return lines


if __name__ == "__main__":
    with open(OUT, "w") as f:
        f.write("# Regression snapshot of the oracle's integer outputs (written by\n")
        f.write("# tests/golden/make_oracle_snapshot.py, which calls only oracle/).\n")
        for line in snapshot_lines():
            f.write(line + "\n")
    print("wrote", OUT)
