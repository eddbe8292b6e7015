"""Writes the stored regression tables in this folder. Calls only the CPU oracle.

Run from the repository root:  python tests/golden/make_golden.py
The tables it freezes were first checked against the oracle's pins (published SplitMix64
test vector, permutation uniformity, exactly-c fold, S^T S = c I) in tests/test_oracle_pins.py.
"""

import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import ss1_tables  # noqa: E402

CASES = [
    # (K, N, c, BK, BN, seed): a few small layers and the first blocks of the fp32 workload
    (64, 64, 2, 64, 64, 0),
    (256, 256, 4, 128, 128, 2),
    (512, 256, 8, 256, 128, 3),
    (768, 768, 2, 64, 64, 0),
]


def main():
    out = {"source": "written by tests/golden/make_golden.py from oracle.ss1_tables", "cases": []}
    for K, N, c, BK, BN, seed in CASES:
        h, g = ss1_tables(K, N, c, BK, BN, seed)
        # freeze block (nb=0, kc=0) in full plus the last block's first 16 entries
        out["cases"].append({
            "K": K, "N": N, "c": c, "BK": BK, "BN": BN, "seed": seed,
            "h_nb0_kc0": h[0, :BK].tolist(), "g_nb0_kc0": g[0, :BK].tolist(),
            "h_last16": h[-1, K - BK:K - BK + 16].tolist(), "g_last16": g[-1, K - BK:K - BK + 16].tolist(),
        })
    with open(os.path.join(HERE, "tables_regression.json"), "w") as f:
        f.write("{\n \"source\": %s,\n \"cases\": [\n" % json.dumps(out["source"]))
        f.write(",\n".join("  " + json.dumps(c) for c in out["cases"]) + "\n ]\n}\n")


if __name__ == "__main__":
    main()
