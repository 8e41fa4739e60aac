"""Pure-Python loops of Eq. (1), Eq. (2) and attention, for tiny inputs only.

Every quantity is accumulated element by element in Python floats (IEEE
double), with no numpy reductions, so these functions check the vectorised
oracle by a route that shares nothing but the definitions:

* Eq. (1) of "详解DSA": I[t, s] = sum_j w[t, j] * ReLU(q[t, j] . k[s]);
* Eq. (2): the k positions of largest score (ties: lower s first), all of
  them when the row has at most k;
* attention of each head over the selected latent entries with the max-
  subtracted softmax.
"""

from __future__ import annotations

import math


def index_score(q_row, w_row, k_vec):
    """q_row: list of H_I vectors (dequantised), w_row: H_I weights, k_vec: d values."""
    total = 0.0
    for j in range(len(q_row)):
        dot = 0.0
        for d in range(len(k_vec)):
            dot += float(q_row[j][d]) * float(k_vec[d])
        if dot > 0.0:
            total += float(w_row[j]) * dot
    return total


def topk_positions(scores, k):
    n = len(scores)
    if n <= k:
        return list(range(n))
    # selection sort by (score desc, position asc)
    taken = []
    used = [False] * n
    for _ in range(k):
        best = -1
        for s in range(n):
            if used[s]:
                continue
            if best < 0 or scores[s] > scores[best]:
                best = s
        used[best] = True
        taken.append(best)
    return taken


def attend(q_heads, rows, sm_scale, value_dim):
    """q_heads: H lists of D values; rows: selected latent rows (D values each)."""
    outs, lses = [], []
    for q in q_heads:
        logits = []
        for c in rows:
            acc = 0.0
            for d in range(len(q)):
                acc += float(q[d]) * float(c[d])
            logits.append(sm_scale * acc)
        if not logits:
            outs.append([0.0] * value_dim)
            lses.append(-math.inf)
            continue
        m = max(logits)
        e = [math.exp(x - m) for x in logits]
        z = sum(e)
        o = [0.0] * value_dim
        for p, c in zip(e, rows):
            for d in range(value_dim):
                o[d] += (p / z) * float(c[d])
        outs.append(o)
        lses.append(m + math.log(z))
    return outs, lses
