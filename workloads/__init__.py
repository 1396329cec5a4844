"""Seeded synthetic workloads for block-sparse attention.

This module only describes problem shapes and draws seeded random inputs.  It
holds none of the attention arithmetic: both the CPU oracle (tests) and the
CUDA path (tests, bench) take their inputs from here, so they see the same
rounded values.

Input recipe (every config):
  * Q, K, V are drawn i.i.d. N(0, 1) in float32 on the CPU from a
    ``torch.Generator`` seeded per config, multiplied by ``input_scale`` (2.0
    for the softcap workload), then rounded to the config dtype (bf16/fp16).
    The pages benchmark on random tensors, not on a trained model
    (FlexAttention vs SDPA on M1 Max, qiita.com/kiarina/items/255a3c0e6e667ebc3cc0,
    section "検証条件").
  * document ids: either the fixed boundaries 2048 and 5000 of the packed-
    document example (dreaming.press FlexAttention how-to, "Mask 3:
    document-packed"), or a seeded variant with n ~ U{4..16} documents whose
    n-1 distinct cut points are drawn uniformly from 1..L-1.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple

import numpy as np
import torch

MASK_CAUSAL = 0
MASK_SLIDING_WINDOW_CAUSAL = 1
MASK_DOCUMENT_CAUSAL = 2
MASK_BITMAP = 3
# decode against a KV cache (lower-right aligned): full, causal, sliding window
MASK_DECODE_FULL = 4
MASK_DECODE_CAUSAL = 5
MASK_DECODE_SLIDING_WINDOW = 6

SCORE_NONE = 0
SCORE_TANH_SOFTCAP = 1

MASK_NAMES = {MASK_CAUSAL: "causal", MASK_SLIDING_WINDOW_CAUSAL: "sliding_window_causal",
              MASK_DOCUMENT_CAUSAL: "document_causal", MASK_BITMAP: "bitmap",
              MASK_DECODE_FULL: "decode_full", MASK_DECODE_CAUSAL: "decode_causal_lower_right",
              MASK_DECODE_SLIDING_WINDOW: "decode_sliding_window_lower_right"}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    S: int
    D: int
    dtype: torch.dtype
    mask_kind: int
    window: int = 0
    doc_boundaries: Optional[Tuple[int, ...]] = None   # fixed document starts (besides 0)
    doc_seeded: bool = False                           # draw 4..16 documents from the seed
    score_kind: int = SCORE_NONE
    softcap: float = 0.0
    input_scale: float = 1.0
    seed: int = 0
    Hkv: Optional[int] = None   # K/V heads (grouped-query attention); None: H

    @property
    def n_kv_heads(self) -> int:
        return self.Hkv if self.Hkv is not None else self.H

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def dtype_name(self) -> str:
        return {torch.bfloat16: "bf16", torch.float16: "fp16"}[self.dtype]

    def describe(self) -> dict:
        d = {"workload": self.name, "B": self.B, "H": self.H, "L": self.L, "S": self.S,
             "D": self.D, "dtype": self.dtype_name, "mask": MASK_NAMES[self.mask_kind],
             "block": 128, "seed": self.seed}
        if self.mask_kind in (MASK_SLIDING_WINDOW_CAUSAL, MASK_DECODE_SLIDING_WINDOW):
            d["window"] = self.window
        if self.mask_kind == MASK_DOCUMENT_CAUSAL:
            d["documents"] = "seeded 4..16" if self.doc_seeded else list(self.doc_boundaries or ())
        if self.mask_kind == MASK_BITMAP:
            d["bitmap"] = "seeded random block classes (empty / all-set / bits at density 0.5)"
        if self.score_kind == SCORE_TANH_SOFTCAP:
            d["score_mod"] = f"tanh_softcap({self.softcap:g})"
        if self.input_scale != 1.0:
            d["input_scale"] = self.input_scale
        if self.n_kv_heads != self.H:
            d["Hkv"] = self.n_kv_heads
        return d


def _w(name, B, H, L, D, dtype, kind, **kw):
    return Workload(name=name, B=B, H=H, L=L, S=L, D=D, dtype=dtype, mask_kind=kind, **kw)


# The five workload families of the benchmark plan.
C1_CAUSAL_256 = _w("causal_L256_B1_H2_D64_bf16", 1, 2, 256, 64, torch.bfloat16, MASK_CAUSAL, seed=1)
C2_CAUSAL_8192 = _w("causal_L8192_B1_H8_D64_bf16", 1, 8, 8192, 64, torch.bfloat16, MASK_CAUSAL, seed=2)
C2_WINDOWS = tuple(
    _w(f"swa{w}_L8192_B1_H8_D64_bf16", 1, 8, 8192, 64, torch.bfloat16, MASK_SLIDING_WINDOW_CAUSAL,
       window=w, seed=3 + i)
    for i, w in enumerate((64, 256, 1024, 4096)))
C3_SWA256_32K = _w("swa256_L32768_B1_H8_D64_bf16", 1, 8, 32768, 64, torch.bfloat16,
                   MASK_SLIDING_WINDOW_CAUSAL, window=256, seed=7)
C4_DOC_FIXED = _w("doc3_L8192_B1_H16_D64_fp16", 1, 16, 8192, 64, torch.float16,
                  MASK_DOCUMENT_CAUSAL, doc_boundaries=(2048, 5000), seed=8)
C4_DOC_SEEDED = _w("docrand_L8192_B1_H16_D64_fp16", 1, 16, 8192, 64, torch.float16,
                   MASK_DOCUMENT_CAUSAL, doc_seeded=True, seed=9)
C5_SWA1024_SOFTCAP = _w("swa1024_softcap30_L16384_B2_H16_D128_bf16x2", 2, 16, 16384, 128,
                        torch.bfloat16, MASK_SLIDING_WINDOW_CAUSAL, window=1024,
                        score_kind=SCORE_TANH_SOFTCAP, softcap=30.0, input_scale=2.0, seed=10)

ALL = (C1_CAUSAL_256, C2_CAUSAL_8192) + C2_WINDOWS + (C3_SWA256_32K, C4_DOC_FIXED, C4_DOC_SEEDED,
                                                      C5_SWA1024_SOFTCAP)
# A tabulated mask (one bit per pair) at the causal workload's shape.
BITMAP_8192 = _w("bitmap_L8192_B1_H8_D64_bf16", 1, 8, 8192, 64, torch.bfloat16, MASK_BITMAP, seed=12)
# Grouped-query attention: 32 query heads sharing 8 K/V heads (SDPA tutorial, section 5).
GQA_CAUSAL_8192 = _w("gqa_causal_L8192_B1_H32_Hkv8_D64_bf16", 1, 32, 8192, 64, torch.bfloat16,
                     MASK_CAUSAL, seed=13, Hkv=8)

# Decode: one new token per sequence against a 32768-token KV cache, 32 query heads
# over 8 K/V heads, batch 8 (SDPA tutorial, section 4, pitfall 3: L = 1, S = cache).
DECODE_32K = Workload(name="decode_L1_S32768_B8_H32_Hkv8_D128_bf16", B=8, H=32, L=1, S=32768,
                      D=128, dtype=torch.bfloat16, mask_kind=MASK_DECODE_CAUSAL, seed=14, Hkv=8)

# The same cache with 4 new tokens per sequence (speculative decoding): 16 query
# rows per K/V head.
DECODE_32K_L4 = Workload(name="decode_L4_S32768_B8_H32_Hkv8_D128_bf16", B=8, H=32, L=4, S=32768,
                         D=128, dtype=torch.bfloat16, mask_kind=MASK_DECODE_CAUSAL, seed=15, Hkv=8)

# 8 new tokens: 32 query rows per K/V head, the most one decode call takes.
DECODE_32K_L8 = Workload(name="decode_L8_S32768_B8_H32_Hkv8_D128_bf16", B=8, H=32, L=8, S=32768,
                         D=128, dtype=torch.bfloat16, mask_kind=MASK_DECODE_CAUSAL, seed=16, Hkv=8)

EXTRA = (BITMAP_8192, GQA_CAUSAL_8192, DECODE_32K, DECODE_32K_L4, DECODE_32K_L8)
BY_NAME = {w.name: w for w in ALL + EXTRA}


def make_qkv(w: Workload, device="cpu"):
    """Seeded Q (B,H,L,D), K, V (B,Hkv,S,D) in the workload dtype, contiguous."""
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    out = []
    hk = w.n_kv_heads
    for shape in ((w.B, w.H, w.L, w.D), (w.B, hk, w.S, w.D), (w.B, hk, w.S, w.D)):
        t = torch.randn(shape, generator=g, dtype=torch.float32)
        if w.input_scale != 1.0:
            t.mul_(w.input_scale)
        out.append(t.to(w.dtype).to(device).contiguous())
    return tuple(out)


def make_doc_id(w: Workload, device="cpu") -> Optional[torch.Tensor]:
    """int32 document id per position (length max(L, S)), or None for other masks."""
    if w.mask_kind != MASK_DOCUMENT_CAUSAL:
        return None
    n = max(w.L, w.S)
    if w.doc_seeded:
        g = torch.Generator(device="cpu").manual_seed(w.seed + 1000)
        ndoc = int(torch.randint(4, 17, (1,), generator=g))
        cuts = torch.randperm(n - 1, generator=g)[: ndoc - 1] + 1
        starts = sorted(int(c) for c in cuts)
    else:
        starts = list(w.doc_boundaries or ())
    return doc_id_from_starts(n, starts, device)


def doc_id_from_starts(n: int, starts, device="cpu") -> torch.Tensor:
    doc = torch.zeros(n, dtype=torch.int32)
    for s in starts:
        doc[s:] += 1
    return doc.to(device)


def random_qkv(B, H, L, S, D, dtype, seed, scale=1.0, device="cpu", Hkv=None):
    """Seeded inputs for an arbitrary (test) shape, same recipe as make_qkv."""
    w = Workload(name="adhoc", B=B, H=H, L=L, S=S, D=D, dtype=dtype, mask_kind=MASK_CAUSAL,
                 input_scale=scale, seed=seed, Hkv=Hkv)
    return make_qkv(w, device)


def random_bitmap(L: int, S: int, seed: int, p_empty: float = 0.35, p_full: float = 0.3,
                  density: float = 0.5) -> np.ndarray:
    """Seeded bitmap mask input: uint32 words (L, 4 * ceil(S / 128)), bit kv % 32 of word
    kv // 32 of row q set when the pair is kept; bits past S are 0.  Each 128 x 128
    block is drawn empty, all-set, or random bits of the given density, so that every
    block class occurs."""
    g = np.random.default_rng(seed)
    nq, nkv = -(-L // 128), -(-S // 128)
    bits = np.zeros((nq * 128, nkv * 128), dtype=bool)
    for i in range(nq):
        for j in range(nkv):
            u = g.random()
            blk = bits[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
            if u < p_empty:
                continue
            if u < p_empty + p_full:
                blk[:] = True
            else:
                blk[:] = g.random((128, 128)) < density
    bits = bits[:L]
    bits[:, S:] = False
    words = np.packbits(bits.reshape(L, -1, 32)[:, :, ::-1], axis=2, bitorder="big")
    return words.view(">u4").reshape(L, nkv * 4).astype(np.uint32)


def make_bitmap(w: Workload) -> Optional[np.ndarray]:
    """The bitmap input of a tabulated-mask workload (uint32 words), else None."""
    if w.mask_kind != MASK_BITMAP:
        return None
    return random_bitmap(w.L, w.S, w.seed)
