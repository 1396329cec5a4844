"""Grouped-query attention on the GPU (query heads sharing K/V heads), against the
fp64 CPU oracle, and bit-for-bit against the same forward on K/V heads repeated
to one per query head."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import masks as OM
from parity import check_workload, compare, oracle_rows, run_gpu, sample_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,Hkv,L,S,D,kind", [
    (2, 4, 2, 300, 300, 64, OM.CAUSAL), (1, 6, 1, 333, 500, 64, OM.SLIDING_WINDOW_CAUSAL),
    (1, 8, 4, 257, 257, 128, OM.DOCUMENT_CAUSAL), (2, 4, 1, 200, 300, 128, OM.BITMAP)])
def test_gqa_all_rows(B, H, Hkv, L, S, D, kind):
    q, k, v = W.random_qkv(B, H, L, S, D, torch.bfloat16, seed=H * 10 + Hkv, Hkv=Hkv)
    window = 100 if kind == OM.SLIDING_WINDOW_CAUSAL else 0
    doc = (torch.randint(0, 3, (max(L, S),), generator=torch.Generator().manual_seed(3),
                         dtype=torch.int32) if kind == OM.DOCUMENT_CAUSAL else None)
    words = W.random_bitmap(L, S, seed=5) if kind == OM.BITMAP else None
    out, lse = run_gpu(q, k, v, kind, window, doc, bitmap=words)
    for b in range(B):
        for h in range(H):
            o_ref, l_ref = oracle_rows(q, k, v, b, h, np.arange(L), kind, window, doc,
                                       bitmap=words)
            compare(out[b, h], lse[b, h], o_ref, l_ref, f"b{b} h{h}")


def test_gqa_equals_repeated_heads_bit_for_bit():
    """Sharing K/V heads changes only which tile is loaded, not the arithmetic."""
    q, k, v = W.random_qkv(1, 8, 1000, 1000, 64, torch.bfloat16, seed=41, Hkv=2)
    og, lg = run_gpu(q, k, v, OM.SLIDING_WINDOW_CAUSAL, 300)
    kr, vr = k.repeat_interleave(4, dim=1), v.repeat_interleave(4, dim=1)
    om, lm = run_gpu(q, kr, vr, OM.SLIDING_WINDOW_CAUSAL, 300)
    assert torch.equal(og, om) and torch.equal(lg, lm)


def test_gqa_32_heads_over_8_sampled():
    w = W.GQA_CAUSAL_8192
    rows = sample_rows(w.L, seed=7)
    check_workload(w, heads=[(0, 0), (0, 5), (0, 31)], rows=rows)


def test_gqa_rejects_uneven_groups():
    import block_sparse_attention_create_b200 as fa
    q = torch.zeros(1, 6, 128, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 4, 128, 64, dtype=torch.bfloat16, device="cuda")
    bm = fa.create_block_mask(0, 128, 128, device="cuda")
    with pytest.raises(ValueError):
        fa.flex_attention(q, k, k, bm)
