"""128x128 block tables by evaluating the mask on every pair.

FlexAttention groups the work into 128x128 token blocks and skips the blocks
that are entirely masked (FlexAttention vs SDPA on M1 Max,
qiita.com/kiarina/items/255a3c0e6e667ebc3cc0, "役割とデータの流れ"; the
how-to's "The two mistakes..." notes only fully masked blocks can be
skipped).  The how-to's create_block_mask(fn, B=None, H=None, Q_LEN, KV_LEN)
broadcasts one mask over batch and heads ("Mask 1: causal").

Classification of block (i, j) over the pairs q in [128 i, 128 i + 127],
kv in [128 j, 128 j + 127]:
  EMPTY   -- no pair is allowed;
  FULL    -- every one of the 128 x 128 pairs is in range and allowed;
  PARTIAL -- otherwise.
A position past Q_LEN or KV_LEN is never allowed, so a block that holds one
is never FULL (reading of a point the pages leave open).

Tables (reading of the FlexAttention BlockMask layout the how-to returns):
``kv_num_blocks[i]`` / ``kv_indices[i, :]`` list the PARTIAL blocks of row i
in ascending j; ``full_kv_num_blocks`` / ``full_kv_indices`` the FULL ones;
unused entries are 0.
"""
from __future__ import annotations

import numpy as np

from . import masks

BLOCK = 128


def classify(kind, q_len, kv_len, window=None, doc_id=None, block=BLOCK, bitmap=None):
    """Return (live, full) bool arrays of shape (nQ, nKV) and allowed-pair count."""
    nq = -(-q_len // block)
    nkv = -(-kv_len // block)
    doc = None if doc_id is None else np.asarray(doc_id, dtype=np.int64)
    live = np.zeros((nq, nkv), dtype=bool)
    full = np.zeros((nq, nkv), dtype=bool)
    allowed_pairs = 0
    padded = np.zeros((block, nkv * block), dtype=bool)
    for i in range(nq):
        rows = np.arange(i * block, min((i + 1) * block, q_len))
        padded[:] = False
        if kv_len > 0:
            m = masks.mask_rows(kind, rows, kv_len, window, doc, bitmap)
            padded[: len(rows), :kv_len] = m
            allowed_pairs += int(m.sum())
        blk = padded.reshape(block, nkv, block)
        live[i] = blk.any(axis=(0, 2))
        full[i] = blk.all(axis=(0, 2))
    return live, full, allowed_pairs


def block_tables(kind, q_len, kv_len, window=None, doc_id=None, block=BLOCK, bitmap=None):
    """Integer tables as int32 numpy arrays (partial and full lists kept apart)."""
    live, full, pairs = classify(kind, q_len, kv_len, window, doc_id, block, bitmap)
    partial = live & ~full
    nq, nkv = live.shape
    kv_num = partial.sum(axis=1).astype(np.int32)
    full_num = full.sum(axis=1).astype(np.int32)
    kv_idx = np.zeros((nq, nkv), dtype=np.int32)
    full_idx = np.zeros((nq, nkv), dtype=np.int32)
    for i in range(nq):
        pj = np.nonzero(partial[i])[0]
        fj = np.nonzero(full[i])[0]
        kv_idx[i, : len(pj)] = pj
        full_idx[i, : len(fj)] = fj
    return {"kv_num_blocks": kv_num, "kv_indices": kv_idx,
            "full_kv_num_blocks": full_num, "full_kv_indices": full_idx,
            "allowed_pairs": pairs, "n_q_blocks": nq, "n_kv_blocks": nkv}


def densities(kind, q_len, kv_len, window=None, doc_id=None, block=BLOCK, bitmap=None):
    """(token density, block density): allowed pairs / all pairs, live blocks / all blocks."""
    live, _, pairs = classify(kind, q_len, kv_len, window, doc_id, block, bitmap)
    return pairs / float(q_len * kv_len), live.sum() / float(live.size)


def transpose(tables):
    """Column view of the tables (FlexAttention's BlockMask also carries it, for
    the backward pass): per kv block j, the q blocks i whose block (i, j) is
    PARTIAL, ascending (``q_num_blocks[j]``, ``q_indices[j, :]``), and those whose
    block is FULL (``full_q_num_blocks``, ``full_q_indices``); unused entries 0."""
    nq, nkv = tables["n_q_blocks"], tables["n_kv_blocks"]
    partial = np.zeros((nq, nkv), dtype=bool)
    full = np.zeros((nq, nkv), dtype=bool)
    for i in range(nq):
        partial[i, tables["kv_indices"][i, : tables["kv_num_blocks"][i]]] = True
        full[i, tables["full_kv_indices"][i, : tables["full_kv_num_blocks"][i]]] = True
    q_num = partial.sum(axis=0).astype(np.int32)
    full_q_num = full.sum(axis=0).astype(np.int32)
    q_idx = np.zeros((nkv, nq), dtype=np.int32)
    full_q_idx = np.zeros((nkv, nq), dtype=np.int32)
    for j in range(nkv):
        pi = np.nonzero(partial[:, j])[0]
        fi = np.nonzero(full[:, j])[0]
        q_idx[j, : len(pi)] = pi
        full_q_idx[j, : len(fi)] = fi
    return {"q_num_blocks": q_num, "q_indices": q_idx,
            "full_q_num_blocks": full_q_num, "full_q_indices": full_q_idx}
