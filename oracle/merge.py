"""fp64 oracle for merging decode results over disjoint parts of the KV:
TEST INFRASTRUCTURE (imported only by tests/ and bench.py's reference legs).

Split-KV merge (not printed on the pages; it belongs to the split-KV form of
the decode path): for one query row whose keys are split into disjoint parts
i with softmax outputs O_i and log-sum-exps lse_i over their own keys,

  L* = log sum_i exp(lse_i)   (the log-sum-exp over all keys)
  O  = sum_i exp(lse_i - L*) O_i

because exp(lse_i - L*) is the share of part i in the full softmax
denominator.  A part with no visible key has lse_i = -inf and weight 0; a row
with no visible key anywhere has O = 0 and L* = -inf, the convention the
decode oracle uses for an empty range.
"""
from __future__ import annotations

import numpy as np


def merge_partials(outs, lses):
    """outs [R, rows, d_v], lses [R, rows] -> (out [rows, d_v], lse [rows]), fp64."""
    o = np.asarray(outs, dtype=np.float64)
    l = np.asarray(lses, dtype=np.float64)
    rows = l.shape[1]
    out = np.zeros((rows, o.shape[2]), dtype=np.float64)
    lse = np.full(rows, -np.inf)
    for r in range(rows):
        m = l[:, r].max()
        if m == -np.inf:
            continue
        lstar = m + np.log(np.sum(np.exp(l[:, r] - m)))
        w = np.exp(l[:, r] - lstar)
        out[r] = (w[:, None] * o[:, r, :]).sum(axis=0)
        lse[r] = lstar
    return out, lse
