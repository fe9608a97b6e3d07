"""Writes tests/golden/tiny64_seed0.npz from the fp64 oracle alone.

The stored arrays are a regression fixture for the oracle itself: the 64 x 64
tiny workload (U(-8, 8) weights, unit scales, no clamp, Grams X^T X/256 + 0.01 I)
rounded by the naive mn x mn Kronecker sweep (the trajectory GPTQ-2D must
reproduce: arxivlens "GPTQ-2D: Cubic-Time Two-Sided Adaptive Rounding",
Analysis > Results).  Run from the repository root:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import workloads  # noqa: E402


def main():
    pb = workloads.tiny(0)
    Q, T = oracle.babai_kron_sweep(pb.W, pb.H_L, pb.H_R, pb.scales, pb.bits, pb.clamp)
    loss = oracle.proxy_loss(pb.W, Q, pb.scales, pb.H_L, pb.H_R)
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny64_seed0.npz")
    np.savez_compressed(out, Q=Q.astype(np.int8), T=T, loss=np.float64(loss))
    print(out, "loss", loss)


if __name__ == "__main__":
    main()
