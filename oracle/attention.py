"""Dense fp64 attention over a boolean mask (the oracle proper).

Definition followed (qiita GeneLab_999 SDPA tutorial, section 1
"SDPAとは何か"): Attention(Q, K, V) = softmax(Q K^T / sqrt(E) + B) V, with
B = 0 where the pair is allowed and -inf where it is masked; here "scale"
generalises 1/sqrt(E) (the tutorial's scale keyword).  The tanh softcap of
the FlexAttention how-to ("Bonus: a score_mod for soft-capping") replaces a
score s by c * tanh(s / c); it is applied to the scaled score, before the
mask, and the mask then decides which entries survive.

The computation is dense: every query row is scored against every key, one
chunk of rows at a time (a full 32768 x 32768 score matrix would not fit, the
size problem the SDPA tutorial's section 2 measures), with no block skipping.

Readings (pinned by tests): LSE is log of the softmax denominator in natural
log, lse = max + log(sum exp(s - max)); a row whose every entry is masked
returns out = 0 and lse = -inf (the tutorial's section 4 reports that SDPA
returns 0 rather than NaN for such rows).
"""
from __future__ import annotations

import numpy as np

from . import masks

NONE = 0
TANH_SOFTCAP = 1


def _as_f64(x):
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def attention_head(q, k, v, kind, window=None, doc_id=None, score_kind=NONE, softcap=0.0,
                   scale=None, rows=None, chunk=256, bitmap=None):
    """One (batch, head): q (L,D), k (S,D), v (S,Dv) -> out (R,Dv), lse (R,).

    ``rows`` selects the query rows to evaluate (default: all L); each row's
    result is independent of the others, so a subset is exact.
    """
    q = _as_f64(q)
    k = _as_f64(k)
    v = _as_f64(v)
    L, D = q.shape
    S = k.shape[0]
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(D)
    rows = np.arange(L) if rows is None else np.asarray(rows, dtype=np.int64)
    doc = None if doc_id is None else _as_f64(doc_id).astype(np.int64)
    out = np.zeros((len(rows), v.shape[1]), dtype=np.float64)
    lse = np.full((len(rows),), -np.inf, dtype=np.float64)
    for c0 in range(0, len(rows), chunk):
        r = rows[c0:c0 + chunk]
        s = (q[r] @ k.T) * scale                       # (R, S) scaled scores
        if score_kind == TANH_SOFTCAP:
            s = softcap * np.tanh(s / softcap)
        allowed = masks.mask_rows(kind, r, S, window, doc, bitmap, q_len=L)
        s = np.where(allowed, s, -np.inf)
        m = s.max(axis=1) if S > 0 else np.full((len(r),), -np.inf)
        live = np.isfinite(m)
        if not live.any():
            continue
        sl = s[live]
        ml = m[live]
        p = np.exp(sl - ml[:, None])                   # exp(-inf) = 0 for masked pairs
        den = p.sum(axis=1)
        idx = np.arange(c0, c0 + len(r))[live]
        out[idx] = (p @ v) / den[:, None]
        lse[idx] = ml + np.log(den)
    return out, lse


def kv_head(h, n_head, n_kv_head):
    """K/V head shared by query head h when n_head query heads share n_kv_head K/V
    heads (grouped-query attention, SDPA tutorial section 5: consecutive query
    heads share one K/V head -- 32 clerks sharing 8 shelves, 4 each -- which is
    what enable_gqa does)."""
    if n_head % n_kv_head:
        raise ValueError("the query heads must divide evenly among the K/V heads")
    return h // (n_head // n_kv_head)


def attention(q, k, v, kind, window=None, doc_id=None, score_kind=NONE, softcap=0.0, scale=None,
              rows=None, heads=None, chunk=256, bitmap=None):
    """Batched oracle on q (B,H,L,D), k and v (B,Hkv,S,D), Hkv dividing H.

    ``heads``: optional list of (b, h) pairs to evaluate (default: all).
    Returns dict {(b, h): (out (R,D) fp64, lse (R,) fp64)}.
    """
    B, H, Hkv = q.shape[0], q.shape[1], k.shape[1]
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    res = {}
    for (b, h) in heads:
        g = kv_head(h, H, Hkv)
        res[(b, h)] = attention_head(q[b, h], k[b, g], v[b, g], kind, window, doc_id, score_kind,
                                     softcap, scale, rows, chunk, bitmap)
    return res
