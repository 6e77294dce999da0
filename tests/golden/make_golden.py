"""Write the stored oracle outputs under tests/golden/.

Calls only the oracle and the seeded input generators (never the CUDA
library): regenerate with `python tests/golden/make_golden.py`.
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import workloads  # noqa: E402


def main():
    w = workloads.make("c1_tiny_int8")
    out = oracle.paged_attn(workloads.oracle_view(w))
    path = os.path.join(HERE, "c1_tiny_int8_oracle.txt")
    with open(path, "w") as f:
        f.write("# FP64 oracle output for the tiny INT8 decode workload (seed 1001):\n")
        f.write("# B=2, seqlens_k={37,64}, q_len=1, H=4, Hk=1, D=64, block_size=16.\n")
        f.write("# Written by tests/golden/make_golden.py (oracle only). Shape %s.\n"
                % (list(out.shape),))
        np.savetxt(f, out.reshape(-1, out.shape[-1]), fmt="%.17g")
    print("wrote", path)


if __name__ == "__main__":
    main()
