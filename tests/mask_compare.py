"""End-to-end mask comparison: the GPU's ranked lists and budgets against the
oracle's own, computed from the oracle's fp64 block scores and head masses
(not from the GPU's).  The two sides may disagree only where the pages leave
the choice to rounding:

  near tie        two blocks whose oracle scores differ by at most
                  1e-3 * max(|s|, 1) may come in either order;
  near threshold  a head's budget k may differ from the oracle's only when
                  the GPU's k is still a minimal gamma-prefix of its own
                  last-row list under the oracle's masses, within 1e-4 of
                  gamma.

ProxyAttn blog, "4. ProxyAttn method": Step 1 "Block Ranking" (the shared
ranking of KV blocks per query block) and Step 2 (the per-head budget as a
prefix of that ranking).  Shared by the GPU parity tests; imports nothing
from the CUDA path.
"""
from __future__ import annotations

import numpy as np

TIE_REL = 1e-3
GAMMA_TOL = 1e-4


def row_span(nb: int, qb: int, causal: bool = True):
    if causal:
        o = qb * (qb + 1) // 2
        return o, qb + 1
    return qb * nb, nb


def forced(qb: int) -> int:
    return 1 if qb == 0 else 2


def compare_lists(gpu_rank, ora_rank, ora_scores, rows, nb, causal=True):
    """rows: (b, g, qb) triples.  Asserts every disagreement is a near tie and
    returns (rows differing, positions differing, positions compared)."""
    nrows = npos = tot = 0
    for b, g, qb in rows:
        o, n = row_span(nb, qb, causal)
        gl = np.asarray(gpu_rank[b, g, o:o + n])
        ol = np.asarray(ora_rank[b, g, o:o + n])
        s = np.asarray(ora_scores[b, g, o:o + n], np.float64)
        tot += n
        assert np.array_equal(np.sort(gl), np.sort(ol)), f"row {(b, g, qb)}: not a permutation of the oracle's"
        assert np.array_equal(gl[:forced(qb)], ol[:forced(qb)]), f"row {(b, g, qb)}: forced blocks differ"
        d = np.nonzero(gl != ol)[0]
        if d.size == 0:
            continue
        nrows += 1
        npos += d.size
        sg, so = s[gl[d]], s[ol[d]]
        lim = TIE_REL * np.maximum(np.abs(so), 1.0)
        assert np.all(np.abs(sg - so) <= lim), (
            f"row {(b, g, qb)}: a disagreement that is not a near tie "
            f"(max |ds| {np.abs(sg - so).max():.3e} at positions {d[:8].tolist()})")
    return nrows, npos, tot


def check_budgets(gpu_budget, gpu_rank, ora_budget, ora_mass, heads, H, G, nb, gamma, causal=True):
    """heads: (b, h) pairs.  Asserts the GPU's budget of each is a minimal
    gamma-prefix of the GPU's own last-row list under the oracle's masses, up
    to GAMMA_TOL; returns how many differ from the oracle's own budget."""
    o, n = row_span(nb, nb - 1, causal)
    F = forced(nb - 1)
    ndiff = 0
    for b, h in heads:
        g = h * G // H
        last = np.asarray(gpu_rank[b, g, o:o + n])
        cum = np.concatenate([[0.0], np.cumsum(np.asarray(ora_mass[b, h], np.float64)[last])])
        k = int(gpu_budget[b, h])
        assert F <= k <= n, (b, h, k)
        assert k == n or cum[k] >= gamma - GAMMA_TOL, f"head {(b, h)}: budget {k} reaches only {cum[k]:.6f}"
        assert k == F or cum[k - 1] < gamma + GAMMA_TOL, f"head {(b, h)}: budget {k} not minimal ({cum[k - 1]:.6f})"
        if k != int(ora_budget[b, h]):
            ndiff += 1
    return ndiff


def log_counts(record: dict):
    """Append one JSON line to $PA_PARITY_LOG (when set) and print it."""
    import json
    import os
    line = json.dumps(record)
    print(line)
    p = os.environ.get("PA_PARITY_LOG")
    if p:
        with open(p, "a") as f:
            f.write(line + "\n")
