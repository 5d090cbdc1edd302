"""Writes the stored expected values under tests/golden/ from the oracle alone.

Run from the repository root:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import nf4  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))


def main():
    c32 = nf4.codebook_f32()
    with open(os.path.join(HERE, "nf4_codebook_f32.txt"), "w") as f:
        f.write("# NF4 codebook, fp32 bit patterns (hex) then value; ascending code 0..15.\n")
        f.write("# Construction: 4-bit NormalFloat (asymmetric N(0,1) quantiles, exact zero,\n")
        f.write("# normalised to [-1, 1]) as read from 'Unsloth vs QLoRA vs Liger-Kernel',\n")
        f.write("# FAQ 'What is the difference between LoRA and QLoRA?'.  Written by\n")
        f.write("# tests/golden/make_golden.py from oracle/nf4.py.\n")
        for v in c32:
            f.write(f"{int(np.float32(v).view(np.uint32)):08x} {float(v):.9g}\n")


if __name__ == "__main__":
    main()
