"""Pure-Python loops over single pairs, for tiny shapes only.

No numpy arithmetic: each score is a Python float sum, each exponential a
math.exp call.  Same definitions as ``attention`` and ``blockmask``
(SDPA tutorial section 1 for the attention; FlexAttention how-to for the masks
and the softcap) written without any vectorisation, to catch an indexing or
broadcasting slip in the vectorised oracle.
"""
from __future__ import annotations

import math


def allowed(kind, q, kv, window=None, doc=None, bitmap=None, q_len=None, kv_len=None):
    if kind == 3:  # tabulated mask_mod: bit kv % 32 of word kv // 32 of row q
        return (int(bitmap[q][kv // 32]) >> (kv % 32)) & 1 == 1
    if kind in (4, 5, 6):  # decode: query q sits at position q + kv_len - q_len
        pos = q + kv_len - q_len
        return kind == 4 or (pos >= kv and (kind == 5 or pos - kv < window))
    if kind == 0:
        return q >= kv
    if kind == 1:
        return q >= kv and q - kv < window
    if kind == 2:
        return q >= kv and doc[q] == doc[kv]
    raise ValueError(kind)


def attention_head(q, k, v, kind, window=None, doc=None, score_kind=0, softcap=0.0, scale=None,
                   bitmap=None):
    """q, k, v: lists of lists of floats. Returns (out rows, lse list)."""
    L, D = len(q), len(q[0])
    S = len(k)
    Dv = len(v[0]) if S else D
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(D)
    outs, lses = [], []
    for i in range(L):
        scores = []
        for j in range(S):
            if not allowed(kind, i, j, window, doc, bitmap, L, S):
                continue
            s = 0.0
            for d in range(D):
                s += q[i][d] * k[j][d]
            s *= scale
            if score_kind == 1:
                s = softcap * math.tanh(s / softcap)
            scores.append((j, s))
        if not scores:
            outs.append([0.0] * Dv)
            lses.append(-math.inf)
            continue
        mx = max(s for _, s in scores)
        den = 0.0
        acc = [0.0] * Dv
        for j, s in scores:
            w = math.exp(s - mx)
            den += w
            for d in range(Dv):
                acc[d] += w * v[j][d]
        outs.append([a / den for a in acc])
        lses.append(mx + math.log(den))
    return outs, lses


def classify_block(kind, i, j, q_len, kv_len, window=None, doc=None, block=128, bitmap=None):
    """'empty' / 'full' / 'partial' for block (i, j) by visiting each pair."""
    n_live = 0
    for q in range(i * block, (i + 1) * block):
        for kv in range(j * block, (j + 1) * block):
            if q < q_len and kv < kv_len and allowed(kind, q, kv, window, doc, bitmap):
                n_live += 1
    if n_live == 0:
        return "empty"
    if n_live == block * block:
        return "full"
    return "partial"
