"""Merge of attention results computed over disjoint key sets -- fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages name the uses of this step without writing it out: "Core 注意力"
("选择最窄的入口": context-parallel attention) and "MLA Prefill" (parameter
table, calcType RING) both split one row's keys over several pieces of work.
The merge follows from the softmax definition alone.  For a query row whose
keys are split into disjoint sets K_1 .. K_S, with x_j the scaled (and masked)
score of key j,

    lse_s = ln sum_{j in K_s} exp(x_j)          out_s = sum_{j in K_s} exp(x_j - lse_s) v_j

so the softmax over all keys has the normaliser sum_s exp(lse_s):

    lse = ln sum_s exp(lse_s)                   out = sum_s exp(lse_s - lse) out_s.

A set with no visible key has lse_s = -inf and weight 0.  A row with no
visible key in any set is 0 with lse -inf, the same reading the forward takes
for an empty row.  The largest lse_s is subtracted before exponentiating (a
shift that cancels in the ratio) so that large scores do not overflow.
"""
from __future__ import annotations

import numpy as np

# Planted mistakes for the pin tests (0 = faithful).
MERGE_PLANTS = {
    1: "weights not divided by their sum",
    2: "merged lse is the max of the parts instead of their log-sum-exp",
    3: "parts weighted equally, ignoring their lse",
}


def merge(outs, lses, *, plant: int = 0):
    """outs: [S, ..., Dv], lses: [S, ...] (natural log).  Returns (out, lse) in fp64."""
    outs = np.asarray(outs, dtype=np.float64)
    lses = np.asarray(lses, dtype=np.float64)
    if outs.shape[:-1] != lses.shape:
        raise ValueError(f"parts {outs.shape} and lse {lses.shape} do not match")
    top = lses.max(axis=0)                                  # [...]
    empty = top == -np.inf
    shift = np.where(empty, 0.0, top)
    w = np.exp(lses - shift)                                # exp(-inf) = 0
    if plant == 3:
        w = np.where(lses == -np.inf, 0.0, 1.0)
    total = w.sum(axis=0)
    safe = np.where(empty, 1.0, total)
    num = (w[..., None] * outs).sum(axis=0)
    out = num if plant == 1 else num / safe[..., None]
    out = np.where(empty[..., None], 0.0, out)
    lse = top if plant == 2 else np.where(empty, -np.inf, shift + np.log(safe))
    return out, lse
