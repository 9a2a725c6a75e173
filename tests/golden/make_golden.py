"""Writes the golden regression fixtures in this folder. Calls only the oracle.

    python tests/golden/make_golden.py

tiny_forward_seed0.txt: sampled outputs of the fp32 forward workload B=1, T=64, C=128
(seed 0; recipe in wkv_inputs.py), computed by the oracle's O(T^2) parallel form of the
wkv equation (concept page "RWKV（Receptance Weighted Key Value）概念", section 3.2) with
the receptance gate.
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import wkv_inputs  # noqa: E402


def main():
    x = wkv_inputs.tiny_forward(seed=0)
    y = oracle.wkv_direct(x.w, x.u, x.k, x.v, x.r)
    g = np.random.Generator(np.random.PCG64(7))
    picks = sorted({(0, int(t), int(c)) for t, c in zip(g.integers(0, 64, 40),
                                                         g.integers(0, 128, 40))})
    picks += [(0, 0, 0), (0, 63, 127), (0, 1, 5)]
    with open(os.path.join(HERE, "tiny_forward_seed0.txt"), "w") as f:
        f.write("# b t c y  -- oracle parallel form, fp32 forward B=1 T=64 C=128 seed 0\n")
        for b, t, c in picks:
            f.write(f"{b} {t} {c} {y[b, t, c]:.17e}\n")


if __name__ == "__main__":
    main()
