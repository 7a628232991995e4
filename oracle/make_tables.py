"""Write ``workloads/tables.json``: seeded per-layer (anchor, d, b) tables.

Test infrastructure: uses only the oracle's cost function (``oracle.bits_per_token``,
``oracle.c0_bits``).  Run ``python oracle/make_tables.py`` to regenerate.

Generator (seeded, deterministic), written from the budgeted action space of the
KV-Kaizen pages ("Action Space and Cost Model"):
  1. every layer starts as an anchor with the least compressed action (d = max, b = max);
  2. while the plan's bits per token exceed the budget C_0 / rho*, pick a layer at random
     and step it down one notch: with probability 0.1 (l > 0) it becomes "inherit",
     otherwise it lowers b by one level (probability 0.7 when both are possible) or d by
     one level; a layer at the lowest (d, b) becomes "inherit" (l > 0);
  3. the anchor map points every inheriting layer at the nearest anchor before it.
A budget that the least compressed plan already meets gives that plan unchanged.
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
sys.path[:] = [x for x in sys.path if os.path.abspath(x or '.') != _HERE]
sys.path.insert(0, os.path.dirname(_HERE))

from oracle import oracle  # noqa: E402
from workloads import TABLES_PATH, WORKLOADS  # noqa: E402


def anchor_map(is_anchor):
    a, cur = [], 0
    for l, f in enumerate(is_anchor):
        if f:
            cur = l
        a.append(cur)
    return a


def generate(n_layers, d_set, b_set, d_rope, budget_bits, seed):
    rng = np.random.default_rng(seed)
    d_set, b_set = sorted(d_set), sorted(b_set)
    is_anchor = [True] * n_layers
    d = [d_set[-1]] * n_layers
    b = [b_set[-1]] * n_layers

    def cost():
        a = anchor_map(is_anchor)
        return oracle.bits_per_token(a, [x if f else 0 for x, f in zip(d, is_anchor)],
                                     [x if f else 0 for x, f in zip(b, is_anchor)], d_rope)

    while cost() > budget_bits:
        l = int(rng.integers(n_layers))
        if not is_anchor[l]:
            continue
        if l > 0 and rng.random() < 0.1:
            is_anchor[l] = False
            continue
        can_b = b[l] > b_set[0]
        can_d = d[l] > d_set[0]
        if can_b and (not can_d or rng.random() < 0.7):
            b[l] = b_set[b_set.index(b[l]) - 1]
        elif can_d:
            d[l] = d_set[d_set.index(d[l]) - 1]
        elif l > 0:
            is_anchor[l] = False
    a = anchor_map(is_anchor)
    dd = [x if f else 0 for x, f in zip(d, is_anchor)]
    bb = [x if f else 0 for x, f in zip(b, is_anchor)]
    return {"anchor": a, "d": dd, "b": bb, "bits_per_token": cost()}


def main():
    out = {}
    for name, w in WORKLOADS.items():
        if not w.budgets:
            continue
        c0 = oracle.c0_bits(w.n_layers, w.n_kv, w.d_h)
        for rho in w.budgets:
            budget = c0 // rho
            t = generate(w.n_layers, w.d_set, w.b_set, w.d_rope, budget, w.seed * 100 + rho)
            t.update({"budget_bits": budget, "c0_bits": c0, "rho_target": rho,
                      "rho": c0 / t["bits_per_token"]})
            out[f"{name}@{rho}x"] = t
    with open(TABLES_PATH, "w") as f:
        json.dump(out, f, indent=1)
    for k, v in out.items():
        n_anchor = sum(1 for l, a in enumerate(v["anchor"]) if a == l)
        print(f"{k:16s} anchors={n_anchor:2d} bits/token={v['bits_per_token']:7d} "
              f"budget={v['budget_bits']:7d} rho={v['rho']:.2f} b-mix={sorted(set(v['b']))}")


if __name__ == "__main__":
    main()
