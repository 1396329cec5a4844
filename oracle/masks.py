"""Mask rules of the FlexAttention how-to, evaluated on index arrays.

Source: "FlexAttention on Apple Silicon: block mask how-to"
(dreaming.press/posts/flexattention-apple-silicon-block-mask-how-to.html):
  * "Mask 1: causal"               -- a query sees keys at or before it.
  * "Mask 2: sliding-window causal" -- causal AND q_idx - kv_idx < W.
  * "Mask 3: document-packed"       -- causal AND document_id[q] == document_id[kv].
  * a tabulated mask_mod (the how-to's create_block_mask takes any function of
    (b, h, q_idx, kv_idx); "Mask 1: causal" shows the form) -- one bit per pair.
  * decode against a KV cache (SDPA tutorial, section 4, pitfall 3): L new
    queries after S - L cached keys see causally aligned to the lower right,
    q_idx + S - L >= kv_idx (torch's causal_lower_right), optionally within a
    window of W keys; or no mask at all.
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
BITMAP = 3
# decode against a KV cache (lower-right alignment; need the query length L)
DECODE_FULL = 4
DECODE_CAUSAL = 5
DECODE_SLIDING_WINDOW = 6


def causal(q_idx, kv_idx):
    return q_idx >= kv_idx


def sliding_window_causal(q_idx, kv_idx, window):
    return (q_idx >= kv_idx) & (q_idx - kv_idx < window)


def document_causal(q_idx, kv_idx, doc_id):
    return (q_idx >= kv_idx) & (doc_id[q_idx] == doc_id[kv_idx])


def bitmap_bits(words, q_idx, kv_idx):
    """Tabulated mask_mod: bit kv % 32 (least significant first) of word kv // 32 of
    row q.  ``words`` is a (Q_LEN, W) uint32 array, W >= ceil(KV_LEN / 32)."""
    w = np.asarray(words, dtype=np.uint32)[q_idx, kv_idx >> 5]
    return ((w >> (kv_idx & 31).astype(np.uint32)) & np.uint32(1)).astype(bool)


def to_bitmap(kind, q_len, kv_len, window=None, doc_id=None, words_per_row=None):
    """Tabulate a mask rule into the bitmap form (rows padded to ``words_per_row``
    words; bits past kv_len are 0)."""
    W = words_per_row if words_per_row is not None else -(-kv_len // 32)
    words = np.zeros((q_len, W), dtype=np.uint32)
    if q_len == 0 or kv_len == 0:
        return words
    m = mask_rows(kind, np.arange(q_len), kv_len, window, doc_id)
    padded = np.zeros((q_len, W * 32), dtype=np.uint64)
    padded[:, :kv_len] = m
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    words[:] = (padded.reshape(q_len, W, 32) * weights).sum(axis=2).astype(np.uint32)
    return words


def causal_lower_right(q_idx, kv_idx, q_len, kv_len):
    return q_idx + (kv_len - q_len) >= kv_idx


def sliding_window_lower_right(q_idx, kv_idx, q_len, kv_len, window):
    pos = q_idx + (kv_len - q_len)   # the query's position in the key sequence
    return (pos >= kv_idx) & (pos - kv_idx < window)


def mask_rows(kind, q_rows, kv_len, window=None, doc_id=None, bitmap=None, q_len=None):
    """Dense boolean mask for the given query rows against keys 0..kv_len-1
    (``q_len``: the number of queries, needed by the decode kinds).

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
    if kind == BITMAP:
        if bitmap is None:
            raise ValueError("bitmap mask needs the bitmap")
        return bitmap_bits(bitmap, q, kv)
    if kind in (DECODE_FULL, DECODE_CAUSAL, DECODE_SLIDING_WINDOW):
        if q_len is None:
            raise ValueError("decode masks need the query length")
        if kind == DECODE_FULL:
            return np.ones((q.shape[0], kv_len), dtype=bool)
        if kind == DECODE_CAUSAL:
            return causal_lower_right(q, kv, q_len, kv_len)
        if window is None:
            raise ValueError("sliding-window mask needs a window")
        return sliding_window_lower_right(q, kv, q_len, kv_len, int(window))
    raise ValueError(f"unknown mask kind {kind}")
