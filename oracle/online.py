"""Tiled online softmax: the same attention by a running max and running sum.

The FlashAttention explainer (service-dock.com/media/flash-attention, third
section, the table of tile sizes 16..1024 over 4096 values) and the
FlashAttention-2 article (media.tcdigital.jp, "分割統治法（Tiling）による
SRAM活用") describe visiting the keys tile by tile while keeping only the
running maximum and the running sum of exponentials, then reconciling at the
end; the explainer states the result equals the plain softmax up to rounding.

This routine is an independent derivation used only to cross-check
``attention.attention_head``: for each key tile it updates
    m' = max(m, max_tile s),  l' = l * exp(m - m') + sum exp(s - m'),
    acc' = acc * exp(m - m') + exp(s - m') @ V_tile,
and returns acc / l and m + log l.
"""
from __future__ import annotations

import numpy as np

from . import masks
from .attention import TANH_SOFTCAP, _as_f64


def attention_head_tiled(q, k, v, kind, window=None, doc_id=None, score_kind=0, softcap=0.0,
                         scale=None, rows=None, tile=128, bitmap=None):
    q = _as_f64(q)
    k = _as_f64(k)
    v = _as_f64(v)
    L, D = q.shape
    S = k.shape[0]
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(D)
    rows = np.arange(L) if rows is None else np.asarray(rows, dtype=np.int64)
    doc = None if doc_id is None else _as_f64(doc_id).astype(np.int64)
    R = len(rows)
    m = np.full((R,), -np.inf)
    l = np.zeros((R,))
    acc = np.zeros((R, v.shape[1]))
    qr = q[rows]
    for t0 in range(0, S, tile):
        t1 = min(S, t0 + tile)
        s = (qr @ k[t0:t1].T) * scale
        if score_kind == TANH_SOFTCAP:
            s = softcap * np.tanh(s / softcap)
        allowed = masks.mask_rows(kind, rows, S, window, doc, bitmap)[:, t0:t1]
        s = np.where(allowed, s, -np.inf)
        m_new = np.maximum(m, s.max(axis=1))
        # rows with no live entry so far keep m = -inf and contribute nothing
        safe = np.where(np.isfinite(m_new), m_new, 0.0)
        alpha = np.where(np.isfinite(m), np.exp(m - safe), 0.0)
        p = np.exp(s - safe[:, None])
        l = l * alpha + p.sum(axis=1)
        acc = acc * alpha[:, None] + p @ v[t0:t1]
        m = m_new
    out = np.zeros_like(acc)
    lse = np.full((R,), -np.inf)
    live = l > 0
    out[live] = acc[live] / l[live, None]
    lse[live] = m[live] + np.log(l[live])
    return out, lse


def softmax_tiled_1d(x, tile):
    """Softmax of a 1-D vector by the running-max / running-sum recurrence."""
    x = np.asarray(x, dtype=np.float64)
    m = -np.inf
    l = 0.0
    for t0 in range(0, len(x), tile):
        xt = x[t0:t0 + tile]
        m_new = max(m, float(xt.max()))
        l = l * np.exp(m - m_new) + float(np.exp(xt - m_new).sum())
        m = m_new
    return np.exp(x - m) / l
