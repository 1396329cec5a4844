"""Mask rules of the FlexAttention how-to, evaluated on index arrays.

Source: "FlexAttention on Apple Silicon: block mask how-to"
(dreaming.press/posts/flexattention-apple-silicon-block-mask-how-to.html):
  * "Mask 1: causal"               -- a query sees keys at or before it.
  * "Mask 2: sliding-window causal" -- causal AND q_idx - kv_idx < W.
  * "Mask 3: document-packed"       -- causal AND document_id[q] == document_id[kv].
True means "this pair is used" (the SDPA boolean-mask convention, qiita
GeneLab_999 SDPA tutorial, section 4, pitfall 1).  Indices are absolute
positions, so for L != S the causal diagonal is upper-left aligned (SDPA
tutorial, section 4, pitfall 3, describes is_causal that way).
"""
from __future__ import annotations

import numpy as np

CAUSAL = 0
SLIDING_WINDOW_CAUSAL = 1
DOCUMENT_CAUSAL = 2


def causal(q_idx, kv_idx):
    return q_idx >= kv_idx


def sliding_window_causal(q_idx, kv_idx, window):
    return (q_idx >= kv_idx) & (q_idx - kv_idx < window)


def document_causal(q_idx, kv_idx, doc_id):
    return (q_idx >= kv_idx) & (doc_id[q_idx] == doc_id[kv_idx])


def mask_rows(kind, q_rows, kv_len, window=None, doc_id=None):
    """Dense boolean mask for the given query rows against keys 0..kv_len-1.

    Returns a bool array of shape (len(q_rows), kv_len).
    """
    q = np.asarray(q_rows, dtype=np.int64)[:, None]
    kv = np.arange(kv_len, dtype=np.int64)[None, :]
    if kind == CAUSAL:
        return causal(q, kv)
    if kind == SLIDING_WINDOW_CAUSAL:
        if window is None:
            raise ValueError("sliding-window mask needs a window")
        return sliding_window_causal(q, kv, int(window))
    if kind == DOCUMENT_CAUSAL:
        if doc_id is None:
            raise ValueError("document mask needs document ids")
        d = np.asarray(doc_id, dtype=np.int64)
        return document_causal(q, kv, d)
    raise ValueError(f"unknown mask kind {kind}")
