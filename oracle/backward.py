"""Gradients of the attention forward (fp64, dense), for the backward pass.

Test infrastructure only, like the rest of oracle/.

The FlashAttention-2 article (media.tcdigital.jp, "あえて再計算して転送を減らす")
describes the backward pass as recomputing the attention matrix on chip from the
saved inputs instead of storing it; what it computes is the derivative of the
forward, written out here from the definition (SDPA tutorial, section 1):

    s = q k^T * scale  (then c * tanh(s / c) under the softcap), masked -> -inf
    P = softmax(s) row by row,  O = P V
    dV = P^T dO
    dP = dO V^T
    dS = P * (dP - rowsum(dO * O))            (softmax backward)
    dS_raw = dS * (1 - tanh(s_scaled / c)^2)  (softcap backward, else dS)
    dQ = dS_raw K * scale,  dK = dS_raw^T Q * scale

A row with no live key has P = 0 and contributes nothing.
"""
from __future__ import annotations

import numpy as np

from . import masks
from .attention import TANH_SOFTCAP, _as_f64


def attention_head_backward(q, k, v, dout, kind, window=None, doc_id=None, score_kind=0,
                            softcap=0.0, scale=None, bitmap=None, return_probs=False):
    """One (batch, head): q (L,D), k (S,D), v (S,Dv), dout (L,Dv) -> dq, dk, dv (fp64);
    with ``return_probs`` also P and dS (both (L,S), dS after the softcap factor),
    for error bounds that need them."""
    q, k, v, dout = (_as_f64(t) for t in (q, k, v, dout))
    L, D = q.shape
    S = k.shape[0]
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(D)
    doc = None if doc_id is None else _as_f64(doc_id).astype(np.int64)
    allowed = masks.mask_rows(kind, np.arange(L), S, window, doc, bitmap, q_len=L)
    t = (q @ k.T) * scale                                  # scaled scores
    s = softcap * np.tanh(t / softcap) if score_kind == TANH_SOFTCAP else t
    s = np.where(allowed, s, -np.inf)
    m = s.max(axis=1, initial=-np.inf) if S > 0 else np.full(L, -np.inf)
    live = np.isfinite(m)
    p = np.zeros_like(s)
    p[live] = np.exp(s[live] - m[live, None])
    p[live] /= p[live].sum(axis=1, keepdims=True)
    out = p @ v
    dv = p.T @ dout
    dp = dout @ v.T
    delta = (dout * out).sum(axis=1, keepdims=True)
    ds = p * (dp - delta)
    if score_kind == TANH_SOFTCAP:
        ds = ds * (1.0 - np.tanh(t / softcap) ** 2)
    dq = ds @ k * scale
    dk = ds.T @ q * scale
    if return_probs:
        return dq, dk, dv, p, ds
    return dq, dk, dv


def attention_head_backward_sampled(q, k, v, dout, kind, q_rows, k_rows, window=None,
                                    doc_id=None, score_kind=0, softcap=0.0, scale=None,
                                    bitmap=None, chunk=256):
    """Exact gradients for a sample of one (batch, head) too large for the dense form:
    dq of the query rows ``q_rows``, dk and dv of the key rows ``k_rows``.

    Each query row's P, dP and dS depend on that row alone (against all keys), and a
    key's dk, dv collect only the rows that see it.  So the rows evaluated are
    q_rows and every query row that sees some key of k_rows, a chunk at a time, by
    the formulas of attention_head_backward.

    Returns a dict: dq (len(q_rows), D), dk and dv (len(k_rows), D) in the given
    orders; rows, the evaluated query rows (ascending); p and ds (len(rows), S), P and
    dS of those rows, for error bounds.
    """
    q, k, v, dout = (_as_f64(t) for t in (q, k, v, dout))
    L, D = q.shape
    S = k.shape[0]
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(D)
    q_rows = np.asarray(q_rows, dtype=np.int64)
    k_rows = np.asarray(k_rows, dtype=np.int64)
    doc = None if doc_id is None else _as_f64(doc_id).astype(np.int64)

    def allowed_of(r):
        return masks.mask_rows(kind, r, S, window, doc, bitmap, q_len=L)

    need = np.zeros(L, dtype=bool)
    need[q_rows] = True
    for c0 in range(0, L, 512):
        r = np.arange(c0, min(L, c0 + 512))
        need[r] |= allowed_of(r)[:, k_rows].any(axis=1)
    rows = np.flatnonzero(need)

    p_all = np.zeros((len(rows), S))
    ds_all = np.zeros((len(rows), S))
    dk = np.zeros((len(k_rows), D))
    dv = np.zeros((len(k_rows), v.shape[1]))
    for c0 in range(0, len(rows), chunk):
        r = rows[c0:c0 + chunk]
        t = (q[r] @ k.T) * scale
        s = softcap * np.tanh(t / softcap) if score_kind == TANH_SOFTCAP else t
        s = np.where(allowed_of(r), s, -np.inf)
        m = s.max(axis=1, initial=-np.inf)
        live = np.isfinite(m)
        p = np.zeros_like(s)
        p[live] = np.exp(s[live] - m[live, None])
        p[live] /= p[live].sum(axis=1, keepdims=True)
        out = p @ v
        delta = (dout[r] * out).sum(axis=1, keepdims=True)
        ds = p * (dout[r] @ v.T - delta)
        if score_kind == TANH_SOFTCAP:
            ds = ds * (1.0 - np.tanh(t / softcap) ** 2)
        p_all[c0:c0 + len(r)] = p
        ds_all[c0:c0 + len(r)] = ds
        dk += ds[:, k_rows].T @ q[r] * scale
        dv += p[:, k_rows].T @ dout[r]
    pos = np.searchsorted(rows, q_rows)
    dq = ds_all[pos] @ k * scale
    return {"dq": dq, "dk": dk, "dv": dv, "rows": rows, "p": p_all, "ds": ds_all}
