"""Pure-Python brute force for decode attention over LOGICAL token lists.

TEST INFRASTRUCTURE ONLY.  It never builds a block pool or reads a block
table: a sequence is simply the list of its tokens' K and V rows in logical
order.  It pins the C oracle's block-table walk (the part a paged layout can
get wrong) on tiny inputs.

Attention is the textbook definition ("PagedAttention and KV memory
management", section "The kernel side": scores, then weighted values), but
written through the log-sum-exp form rather than the max/sum form the C
oracle uses, with exactly rounded sums (math.fsum):

    s_t = scale * <q, k_t>,   lse = log sum_t exp(s_t),
    out = sum_t exp(s_t - lse) * v_t.

Query head h uses kv head h // G with G = Hq // Hkv.  An empty sequence gives
a zero row.
"""
from __future__ import annotations

import math
from typing import Sequence

Row = Sequence[float]


def logsumexp(xs: Sequence[float]) -> float:
    top = max(xs)
    return top + math.log(math.fsum(math.exp(x - top) for x in xs))


def attend_logical(q: Row, keys: Sequence[Row], values: Sequence[Row], scale: float) -> list[float]:
    """One query row against one sequence's logical K and V rows."""
    D = len(q)
    if not keys:
        return [0.0] * D
    scores = [scale * math.fsum(qd * kd for qd, kd in zip(q, k)) for k in keys]
    lse = logsumexp(scores)
    weights = [math.exp(s - lse) for s in scores]
    return [math.fsum(w * v[d] for w, v in zip(weights, values)) for d in range(D)]


def decode_logical(q, keys, values, scale: float):
    """q[b][h] -> D floats; keys[b][t][kvh] / values[b][t][kvh] -> D floats.

    Returns out[b][h] as lists of floats.
    """
    out = []
    for b, q_b in enumerate(q):
        Hq = len(q_b)
        Hkv = len(keys[b][0]) if keys[b] else None
        rows = []
        for h in range(Hq):
            if not keys[b]:
                rows.append([0.0] * len(q_b[h]))
                continue
            G = Hq // Hkv
            kvh = h // G
            ks = [tok[kvh] for tok in keys[b]]
            vs = [tok[kvh] for tok in values[b]]
            rows.append(attend_logical(q_b[h], ks, vs, scale))
        out.append(rows)
    return out


def prefill_logical(q, keys, values, scale: float):
    """Causal multi-query attention over logical lists.

    q[b] is a list of query tokens, each a list over query heads of D floats;
    they are the last len(q[b]) tokens of sequence b (whose keys/values are
    keys[b][t][kvh]).  Query i sits at position L - n + i and sees tokens
    0..that position.  Returns out[b][i][h].
    """
    out = []
    for b, qb in enumerate(q):
        L, n = len(keys[b]), len(qb)
        rows = []
        for i, qtok in enumerate(qb):
            pos = L - n + i
            Hq = len(qtok)
            Hkv = len(keys[b][0])
            G = Hq // Hkv
            rows.append([attend_logical(qtok[h], [tok[h // G] for tok in keys[b][: pos + 1]],
                                        [tok[h // G] for tok in values[b][: pos + 1]], scale) for h in range(Hq)])
        out.append(rows)
    return out
