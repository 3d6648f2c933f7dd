"""Per-element brute force of the FlashPrefill path for tiny inputs (pure Python floats).

TEST INFRASTRUCTURE ONLY (see the package header). Written independently of
``flashprefill_oracle`` -- scalar loops, no numpy arithmetic -- so that the two
can be checked against each other: a dropped term, a wrong index or a
transposed operand in either shows up as a disagreement.

Steps, in the order of the FlashPrefill summary page's Method section (block
mean pooling; dynamic threshold alpha * row max with sink and window blocks
always kept; index compaction), then exact softmax attention of every query
token over the keys of its row's kept blocks that do not lie after it. One
list per KV group: the union over the group's query heads (PackGQA).
"""
from __future__ import annotations

import math


def brute_force(Q, K, V, B, alpha, sink_tokens, window_tokens, scale=None):
    """Q: nested lists [L][Hq][d]; K, V: [L][Hkv][d] (Python floats).

    Returns dict(mask, lists, O, lse) with mask[g][i][j] (bool, j <= i),
    lists[g][i] (ascending), O[t][h][c] and lse[h][t]."""
    L = len(Q)
    Hq = len(Q[0])
    Hkv = len(K[0])
    d = len(Q[0][0])
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    N = (L + B - 1) // B

    def block_tokens(i):
        return list(range(i * B, min(i * B + B, L)))

    def mean_vec(X, i, head):
        toks = block_tokens(i)
        return [sum(X[t][head][c] for t in toks) / len(toks) for c in range(d)]

    qbar = [[mean_vec(Q, i, h) for h in range(Hq)] for i in range(N)]
    kbar = [[mean_vec(K, j, g) for g in range(Hkv)] for j in range(N)]

    n_sink = -(-sink_tokens // B)
    n_win = max(1, -(-window_tokens // B))

    mask = [[[False] * N for _ in range(N)] for _ in range(Hkv)]
    for h in range(Hq):
        g = h // G
        for i in range(N):
            scores = []
            for j in range(i + 1):
                dot = 0.0
                for c in range(d):
                    dot += qbar[i][h][c] * kbar[j][g][c]
                scores.append(scale * dot)
            top = max(scores)
            for j in range(i + 1):
                if math.exp(scores[j] - top) >= alpha:
                    mask[g][i][j] = True
    for g in range(Hkv):
        for i in range(N):
            for j in range(i + 1):
                if j < n_sink or i - j < n_win:
                    mask[g][i][j] = True

    lists = [[[j for j in range(N) if mask[g][i][j]] for i in range(N)] for g in range(Hkv)]

    O = [[[0.0] * d for _ in range(Hq)] for _ in range(L)]
    lse = [[0.0] * L for _ in range(Hq)]
    for t in range(L):
        i = t // B
        for h in range(Hq):
            g = h // G
            keys = [kk for kk in range(t + 1) if mask[g][i][kk // B]]
            logits = []
            for kk in keys:
                dot = 0.0
                for c in range(d):
                    dot += Q[t][h][c] * K[kk][g][c]
                logits.append(scale * dot)
            top = max(logits)
            w = [math.exp(x - top) for x in logits]
            z = sum(w)
            for c in range(d):
                O[t][h][c] = sum(w[n] * V[keys[n]][g][c] for n in range(len(keys))) / z
            lse[h][t] = top + math.log(z)
    return dict(mask=mask, lists=lists, O=O, lse=lse)
