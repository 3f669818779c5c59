"""Writes engram_rows.json: hashed rows of a fixed small token batch under
the Engram hash this library defines ("Conditional Memory via Scalable
Lookup" review, "다중 헤드 해싱" names independent hashes per order and head
without giving them; the definition is the one in include/pkm.h).  It calls
only the oracle.  The stored rows freeze the definition: the GPU parity
tests compare the CUDA path with the oracle, this file keeps the oracle
itself from drifting.

Run from the repository root: python tests/golden/make_engram_rows.py
"""

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402

TOKENS = [[0, 1, 2, 3, 2147483647, 5, 5, 5], [7, 8, 9, 7, 8, 9, 100000, 42]]
ORDERS = [1, 2, 3]
K = 2
SEEDS = [0, 1, 0x9E3779B97F4A7C15, 12345, 2 ** 63, 2 ** 64 - 1]
M = [97, 101, 1048573, 1, 65536, 2147483629]


def main():
    rows = oracle.engram_rows(TOKENS, ORDERS, K, SEEDS, M)
    out = dict(source="Conditional Memory via Scalable Lookup review, multi-head hashing; "
                      "hash as defined in include/pkm.h (pkm_engram_forward)",
               tokens=TOKENS, orders=ORDERS, K=K, seeds=[str(s) for s in SEEDS], M=M,
               rows=rows.tolist())
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "engram_rows.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(path)


if __name__ == "__main__":
    main()
