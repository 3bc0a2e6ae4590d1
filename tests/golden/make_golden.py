"""Write the stored oracle tables under tests/golden/ (calls only the oracle).

    python tests/golden/make_golden.py

nf4_levels.txt: the 16 NF4 levels as fp32 bit patterns.  The pages do not print
the levels ("Can You Fine-Tune a 27B Model on a Laptop?", 2:19-2:29 only names a
4-bit format for bell-curve weights); the oracle builds them by QLoRA's
normal-quantile construction, and this file freezes its output so that a later
change to that construction fails a test instead of passing silently.
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402


def main():
    c = oracle.nf4_codebook()
    with open(os.path.join(HERE, "nf4_levels.txt"), "w") as f:
        f.write("# NF4 levels (index, fp32 bits, value) written by tests/golden/make_golden.py from the oracle.\n")
        f.write("# Construction: QLoRA normal quantiles, p_max = 1 - (1/32 + 1/30)/2, 7 negative + 0 + 8 positive,\n")
        f.write("# normalised to [-1, 1], rounded once to fp32.\n")
        for i, v in enumerate(c):
            f.write(f"{i:2d} {int(np.array(v).view(np.uint32)):08x} {float(v):+.9g}\n")


if __name__ == "__main__":
    main()
