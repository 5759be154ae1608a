"""Write the stored expected values under tests/golden/ from the CPU oracle alone.

Run from the repository root:  python tests/golden/make_golden.py
It builds the seeded tiny fp32 workload (4 sequences, contexts {1, 15, 16, 37}, 4 heads,
head_dim 64, block_size 16, pool of 32 blocks), runs the oracle's step on it (the new tokens'
cache write, then decode) and stores the fp64 output with 17 significant digits.  The vLLM
tutorials print no worked example with numbers, so no stored value comes from them; this file
is a regression record of the oracle, regenerated only when a change to the oracle's
arithmetic is justified by the sources.
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from paged_kv_cache_427_b200 import workloads  # noqa: E402


def main():
    orc = oracle.load()
    b = workloads.tiny_fp32()
    kc, vc = b.key_cache.copy(), b.value_cache.copy()
    assert orc.reshape_and_cache(b.key, b.value, kc, vc, b.slot_mapping, b.dtype) == 0
    out = orc.decode(b.query, kc, vc, b.block_tables, b.context_lens, b.scale, b.dtype)
    path = os.path.join(HERE, "tiny_fp32_oracle.txt")
    with open(path, "w") as f:
        f.write("# oracle output for the tiny fp32 workload, shape [4, 4, 64], C order\n")
        f.write("# written by tests/golden/make_golden.py (calls only oracle/ and the generator)\n")
        for x in out.ravel():
            f.write(f"{x:.17g}\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
