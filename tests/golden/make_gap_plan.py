"""Writes tests/golden/gap_plan.json: the score-gap redraw plan of each workload.

The parity contract compares selected block indices bit for bit.  That is only
a fair test where the k-1-th and k-th ranked block scores of a query block are
more than GAP apart, so that fp32 (the kernel) and fp64 (the oracle) cannot
order them differently.  For every row (b, kvh, query block i) whose fp64
oracle gap is <= GAP at any budget the workload uses, this script bumps the
row's redraw attempt; the generator then replaces that row's query noise with
a draw from PCG64(SeedSequence([seed, b, kvh, i, attempt])).  It repeats until
every row passes (at most 64 attempts per row).

Only the oracle is used to compute gaps.  Run from the repository root:
    python tests/golden/make_gap_plan.py [workload ...]
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import gen  # noqa: E402
import oracle  # noqa: E402

GAP = 1e-3
MAX_ATTEMPTS = 64
PLAN = os.path.join(ROOT, "tests", "golden", "gap_plan.json")


def failing_rows(x: gen.SynthInputs):
    """(b, kvh, i) rows whose gap is <= GAP at any of the workload's budgets."""
    kbar, qbar = oracle.block_pool(x.k, x.q)
    bad = set()
    for topk in x.workload.gap_budgets:
        _, gap = oracle.block_select(qbar, kbar, topk)
        for b, h, i in zip(*np.nonzero(~np.isnan(gap) & (gap <= GAP))):
            bad.add((int(b), int(h), int(i)))
    return bad


def plan_for(name: str):
    attempts = {}
    for _ in range(MAX_ATTEMPTS):
        redraws = [[b, h, i, a] for (b, h, i), a in sorted(attempts.items())]
        x = gen.make_inputs(name, redraws=redraws)
        bad = failing_rows(x)
        if not bad:
            return redraws
        for row in bad:
            attempts[row] = attempts.get(row, 0) + 1
            if attempts[row] > MAX_ATTEMPTS:
                raise RuntimeError(f"{name}: row {row} has no gap after {MAX_ATTEMPTS} redraws")
    raise RuntimeError(f"{name}: plan did not converge")


def main(names):
    data = {}
    if os.path.exists(PLAN):
        with open(PLAN) as f:
            data = json.load(f)
    for name in names:
        w = gen.WORKLOADS[name]
        redraws = plan_for(name)
        data[name] = {"seed": w.seed, "gap": GAP, "budgets": list(w.gap_budgets),
                      "redraws": redraws}
        print(f"{name}: {len(redraws)} rows redrawn")
    with open(PLAN, "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)
        f.write("\n")


if __name__ == "__main__":
    main(sys.argv[1:] or list(gen.WORKLOADS))
