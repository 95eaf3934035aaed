"""Acceptance rule for an indexer top-k result against the oracle (test infrastructure).

For each evaluated query row, with oracle set O (its non -1 indices) and the
candidate set G:

* recall = |G & O| / |O|  (1 when O is empty); mean recall over rows >= 0.999;
* when the row sees at most k keys, G must equal O exactly;
* every j in G but not in O must have an oracle score of at least the oracle's
  k-th score minus ``tol_rel`` * max |oracle score over the row's visible keys|
  (tol_rel = 1e-3);
* G holds no duplicate, no key outside [0, V_t), and exactly min(k, V_t)
  entries, and the candidate's -1 padding comes after its real entries.

The recall-plus-tolerance form follows the set-overlap recall the StreamIndex
abstract reports against the full computation; the 1e-3 bound is the
tolerance stated for this indexer step.
"""

from __future__ import annotations

import numpy as np


def check(rows, V, k, oracle_idx, oracle_score, cand_idx, extra_scores, row_absmax,
          tol_rel: float = 1e-3):
    """Evaluate the rule.

    rows: [n] flat rows; V: [n] visible counts; oracle_idx/oracle_score [n,k];
    cand_idx [n,k] int; extra_scores [n,k]: oracle fp64 score of each
    cand_idx entry (nan where -1); row_absmax [n].
    Returns a dict with mean/min recall, violations and structural errors.
    """
    n = len(rows)
    recalls = np.ones(n)
    violations = []
    struct_err = []
    exact_err = []
    for i in range(n):
        o = oracle_idx[i][oracle_idx[i] >= 0]
        g_row = cand_idx[i]
        nreal = int(min(k, V[i]))
        g = g_row[g_row >= 0]
        if g.size != nreal or np.any(g_row[:nreal] < 0) or np.any(g_row[nreal:] != -1):
            struct_err.append((int(rows[i]), "count/padding"))
        if np.unique(g).size != g.size:
            struct_err.append((int(rows[i]), "duplicate"))
        if g.size and (g.min() < 0 or g.max() >= V[i]):
            struct_err.append((int(rows[i]), "not visible"))
        if o.size:
            recalls[i] = np.intersect1d(g, o).size / o.size
        if V[i] <= k and not np.array_equal(np.sort(g), np.sort(o)):
            exact_err.append(int(rows[i]))
        if o.size and g.size:
            kth = oracle_score[i][o.size - 1]
            bound = kth - tol_rel * row_absmax[i]
            extra = np.setdiff1d(g, o)
            for j in extra:
                pos = np.nonzero(g_row == j)[0][0]
                s = extra_scores[i][pos]
                if not (s >= bound):
                    violations.append((int(rows[i]), int(j), float(s), float(kth)))
    return {
        "rows": n,
        "mean_recall": float(recalls.mean()) if n else 1.0,
        "min_recall": float(recalls.min()) if n else 1.0,
        "violations": violations,
        "struct_errors": struct_err,
        "exact_errors": exact_err,
    }


def passed(res, mean_recall_min: float = 0.999) -> bool:
    return (res["mean_recall"] >= mean_recall_min and not res["violations"]
            and not res["struct_errors"] and not res["exact_errors"])
