"""Writes the golden fixtures of this directory from the oracle alone.

    python tests/golden/make_golden.py

e2m1_identity.txt  : for each of the 16 E2M1 codes, the E4M3 byte that page 1's
                     identity gives for the code in a high nibble, and the two
                     decoded values (the oracle's E2M1 and E4M3 tables).
tiny_w4a4_y_x1024.txt : the tiny W4A4 workload (128 x 256 x 256, seed 0)
                     through the oracle's FP64 product, times 2^10: every value
                     is an integer (doubled codes in [-12, 12], scale exponents
                     in [-4, 4]).  Stored as the SHA-256 of the int64 array and
                     64 sampled (row, col, value) entries.
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from block_scaled_precision_nvfp4_b200 import workloads as wl  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))


def main():
    with open(os.path.join(HERE, "e2m1_identity.txt"), "w") as f:
        f.write("# code e4m3_byte e2m1_value e4m3_value   (written by make_golden.py from the oracle)\n")
        for c in range(16):
            b = oracle.e2m1_to_e4m3_word(c << 4) & 0xFF
            f.write(f"{c} 0x{b:02x} {oracle.e2m1_value(c)!r} {oracle.e4m3_value(b)!r}\n")
    t = wl.tiny_w4a4(0)
    Y = oracle.gemm_w4a4(t.A.codes, t.A.scales, 1.0, t.W.codes, t.W.scales, 1.0, t.M, t.N, t.K)
    Yi = Y * 1024.0
    assert np.array_equal(Yi, np.round(Yi))
    Yi = Yi.astype(np.int64)
    import hashlib
    rng = np.random.default_rng(0)
    idx = rng.integers(0, Yi.size, 64)
    with open(os.path.join(HERE, "tiny_w4a4_y_x1024.txt"), "w") as f:
        f.write("# tiny W4A4 128x256x256 seed 0: oracle Y * 2^10 (written by make_golden.py)\n")
        f.write(f"sha256 {hashlib.sha256(np.ascontiguousarray(Yi).tobytes()).hexdigest()}\n")
        for i in idx:
            r, c = divmod(int(i), Yi.shape[1])
            f.write(f"{r} {c} {Yi[r, c]}\n")


if __name__ == "__main__":
    main()
