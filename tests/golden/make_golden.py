"""Writes the golden fixtures in this folder.  Calls only the CPU oracle.

    python tests/golden/make_golden.py

nf4_codebook_eq2.txt: the 16 NF4 levels of eq. 2 of "QLoRA: Efficient
Fine-Tuning" (q_i = Phi^-1((i - 1/2) / 16)), divided by the largest level and
rounded to fp32, as hex bit patterns, followed by the 15 snapping thresholds.
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import oracle as O  # noqa: E402


def main():
    q = O.nf4_codebook()
    t = O.snap_thresholds(q)
    with open(os.path.join(HERE, "nf4_codebook_eq2.txt"), "w") as f:
        f.write("# NF4 levels: eq. 2 of 'QLoRA: Efficient Fine-Tuning' (Step 1),\n")
        f.write("# q_i = Phi^-1((i - 1/2)/16), i = 1..16, divided by q_16, rounded to fp32.\n")
        f.write("# fp32 hex bits, then the decimal value.  Written by make_golden.py (oracle only).\n")
        for v in q:
            f.write(f"{int(v.view('uint32')):08x}  {float(v):+.9f}\n")
    with open(os.path.join(HERE, "nf4_thresholds.txt"), "w") as f:
        f.write("# Snapping thresholds t_j = smallest fp32 >= (q_j + q_{j+1})/2, j = 0..14,\n")
        f.write("# for the eq. 2 codebook ('snapped to the nearest NF4 quantile level').\n")
        for v in t:
            f.write(f"{int(v.view('uint32')):08x}  {float(v):+.9f}\n")


if __name__ == "__main__":
    main()
