"""Writes the stored expected values under tests/golden/ from the oracle alone.

Run from the repository root:  python tests/golden/make_golden.py
It calls only ``oracle`` (and ``synth`` for seeded inputs), never the CUDA path.
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import nf4  # noqa: E402


def main():
    q = nf4.nf4_codebook()
    with open(os.path.join(HERE, "nf4_codebook.txt"), "w") as f:
        f.write("# NF4 codebook written by tests/golden/make_golden.py from oracle.nf4.nf4_codebook()\n")
        f.write("# (reading R3 of the quantile construction; one fp32 per line as hex bits and decimal)\n")
        for v in q:
            f.write("%08x %.9g\n" % (int(np.float32(v).view(np.uint32)), float(v)))


if __name__ == "__main__":
    main()
