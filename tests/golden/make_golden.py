"""Writes the regression fixtures in this folder.  Calls only the oracle.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402

CASES = [
    # the 32-layer decode workload (N = 1024) and the batched long-context one (N = 2048)
    dict(name="llada32_n1024", N=1024, L=32, rho_p=0.25, l_p=12, rho_1=0.06, rho_L=0.06),
    dict(name="llada32_n2048", N=2048, L=32, rho_p=0.25, l_p=12, rho_1=0.06, rho_L=0.06),
    dict(name="tiny2_uniform", N=64, L=2, rho_p=0.25, l_p=1, rho_1=0.25, rho_L=0.25),
    dict(name="asym_n4096", N=4096, L=28, rho_p=0.3, l_p=9, rho_1=0.02, rho_L=0.1),
]


def main():
    out = {"written_by": "tests/golden/make_golden.py (oracle.budget_table)", "cases": []}
    for c in CASES:
        k = oracle.budget_table(c["N"], c["L"], c["rho_p"], c["l_p"], c["rho_1"], c["rho_L"])
        out["cases"].append(dict(c, k=k))
    with open(os.path.join(HERE, "budget_tables.json"), "w") as fh:
        json.dump(out, fh, indent=1)


if __name__ == "__main__":
    main()
