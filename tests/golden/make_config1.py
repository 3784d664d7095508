"""Writes config1_w4g128.npz: the W4 G128 256 x 1024 matrix fitted by the
oracle's data-free group fitter from i.i.d. Laplace(0, 0.02) FP32 weights
(seed 0).  Calls only oracle/ (and the seeded input generator for the
source weights).

    python tests/golden/make_config1.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle      # noqa: E402
import synthetic   # noqa: E402

N, K, B, G = 256, 1024, 4, 128
OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "config1_w4g128.npz")


def main():
    w = synthetic.laplace_weights(0, N * K, 0.02).numpy().astype(np.float64)
    r = oracle.fit(w, G, B, oracle.MIDRISE)
    codes = r["codes"].reshape(N, K)
    np.savez_compressed(
        OUT, packed=oracle.pack(codes, B), scales=r["s"].reshape(N, K // G),
        ab=r["ab"].reshape(N, K // G, 2), sse=r["sse"], clipped=r["clipped"])
    print(OUT, "NRMSE", oracle.nrmse(r["sse"], w),
          "clipped", r["clipped"].sum() / w.size)


if __name__ == "__main__":
    main()
