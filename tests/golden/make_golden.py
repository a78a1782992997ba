"""Writes tests/golden/tiny_expected.npz from the CPU oracle alone.

Inputs are the seeded tiny workload (X 16x256 ~ N(0,1), W 128x256 ~ N(0,0.02),
seed 0, dynamic per-tensor global scales); the stored arrays are the oracle's
packed codes, logical block scales, global scales and fp64 output.  Run:
    python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from nvfp4_w4a4_block_b200 import workloads as W  # noqa: E402


def main():
    wl = W.TINY
    x, w = wl.x(), wl.w()
    ref = oracle.linear_reference(x, w, wl.seg_offsets)
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_expected.npz")
    np.savez_compressed(out, x=x, w=w, qx=ref["qx"], sfx=ref["sfx"], qw=ref["qw"], sfw=ref["sfw"],
                        s_x=np.float32(ref["s_x"]), s_w=ref["s_w"], y=ref["y"])
    print("wrote", out)


if __name__ == "__main__":
    main()
