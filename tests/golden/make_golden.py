"""Writes the stored expected values under tests/golden/ by calling only the oracle.

    python tests/golden/make_golden.py
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import nf4  # noqa: E402


def main():
    c = nf4.codebook()
    with open(os.path.join(HERE, "nf4_codebook.txt"), "w") as f:
        f.write("# NF4 levels (QLoRA 4-bit NormalFloat with exact zero; see oracle/nf4.py for\n")
        f.write("# the reading of delta). Written by tests/golden/make_golden.py from the oracle.\n")
        f.write("# index fp32_bits value\n")
        for i, x in enumerate(c):
            f.write("%2d 0x%08x % .9e\n" % (i, int(x.view("uint32")), float(x)))


if __name__ == "__main__":
    main()
