"""Writes the stored expected values under tests/golden/ that are too slow
to recompute in every test run.  Calls only the oracle and the seeded input
generators.

gated_T_seed101.npy: BSFA thresholds T[h, i] (fp32, [Hq=32, nQB=512]) for
the gated prefill workload (Llama-3.1-8B attention shape, L = 32768, 64x64
tiles), calibrated on a separate seed (101) of the same synthetic recipe:
the k-th largest (k = 64) off-diagonal block max of q-block i, -inf when
fewer than k candidates exist (Block Sparse Flash Attention, Figure 2a).

Usage: python -m oracle.make_golden
"""
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402
from oracle import sbfa_oracle as O  # noqa: E402

GOLDEN = os.path.join(ROOT, "tests", "golden")


def gated_thresholds(L=32768, Hq=32, Hkv=8, block=64, k_top=64, seed=101):
    wl = W.make_gated(B=1, Hq=Hq, Hkv=Hkv, L=L, block=block, seed=seed)
    G = Hq // Hkv
    n = L // block
    smax = np.full((Hq, n, n), -np.inf)
    for h in range(Hq):
        t = time.time()
        smax[h] = O.block_max_head(wl.q[0, :, h, :], wl.k[0, :, h // G, :], block, wl.scale)
        print(f"  head {h}: {time.time() - t:.1f}s", flush=True)
    return O.calibrate_thresholds(smax, k_top).astype(np.float32)


if __name__ == "__main__":
    T = gated_thresholds()
    np.save(os.path.join(GOLDEN, "gated_T_seed101.npy"), T)
    print("wrote gated_T_seed101.npy", T.shape, np.isfinite(T).sum())
