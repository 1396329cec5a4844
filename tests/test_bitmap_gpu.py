"""Tabulated mask_mod (one bit per pair) and the column (transpose) tables on the
GPU, against the fp64 CPU oracle: block tables bit-exact, forward element by
element within the parity tolerances, and a bitmap that tabulates the causal
rule giving the causal kind's output bit for bit."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import blockmask as OB
from oracle import masks as OM
from parity import bitmap_to_device, compare, oracle_rows, run_gpu, sample_rows

pytestmark = pytest.mark.gpu

TABLE_KEYS = ("kv_num_blocks", "kv_indices", "full_kv_num_blocks", "full_kv_indices")
T_KEYS = ("q_num_blocks", "q_indices", "full_q_num_blocks", "full_q_indices")


def _fa():
    import block_sparse_attention_create_b200 as fa
    return fa


@pytest.mark.parametrize("L,S,seed", [(300, 200, 1), (1000, 1000, 2), (129, 1, 3), (1, 129, 4),
                                      (4096, 2048, 5)])
def test_bitmap_tables_bit_exact(L, S, seed):
    fa = _fa()
    words = W.random_bitmap(L, S, seed)
    bm = fa.create_block_mask(fa.FA_MASK_BITMAP, L, S, bitmap=bitmap_to_device(words))
    torch.cuda.synchronize()
    got = bm.tables()
    ref = OB.block_tables(OM.BITMAP, L, S, bitmap=words)
    for key in TABLE_KEYS:
        assert np.array_equal(got[key].reshape(ref[key].shape), ref[key]), key


@pytest.mark.parametrize("kind,L,S,window", [(0, 8192, 8192, 0), (1, 8192, 8192, 256),
                                             (1, 700, 300, 50), (2, 1000, 1000, 0),
                                             (3, 1000, 700, 0), (0, 5, 300, 0)])
def test_transpose_bit_exact(kind, L, S, window):
    fa = _fa()
    doc = words = None
    if kind == 2:
        doc = torch.randint(0, 4, (max(L, S),), generator=torch.Generator().manual_seed(L),
                            dtype=torch.int32)
    if kind == 3:
        words = W.random_bitmap(L, S, seed=L + S)
    bm = fa.create_block_mask(kind, L, S, window=window,
                              doc_id=doc.cuda() if doc is not None else None,
                              bitmap=bitmap_to_device(words) if words is not None else None)
    t = {k: v.cpu().numpy() for k, v in bm.transpose().items()}
    ref = OB.transpose(OB.block_tables(kind, L, S, window or None,
                                       None if doc is None else doc.numpy(), bitmap=words))
    for key in T_KEYS:
        assert np.array_equal(t[key].reshape(ref[key].shape), ref[key]), key


@pytest.mark.parametrize("L,S,D,dtype,sk", [(300, 200, 64, torch.bfloat16, 0),
                                            (700, 900, 64, torch.float16, 0),
                                            (513, 513, 128, torch.bfloat16, 1),
                                            (257, 640, 128, torch.float16, 0)])
def test_bitmap_forward_all_rows(L, S, D, dtype, sk):
    q, k, v = W.random_qkv(2, 2, L, S, D, dtype, seed=L * 3 + S)
    words = W.random_bitmap(L, S, seed=L + 7 * S)
    cap = 20.0 if sk else 0.0
    out, lse = run_gpu(q, k, v, OM.BITMAP, score_kind=sk, softcap=cap, bitmap=words)
    for b in range(2):
        for h in range(2):
            o_ref, l_ref = oracle_rows(q, k, v, b, h, np.arange(L), OM.BITMAP, score_kind=sk,
                                       softcap=cap, bitmap=words)
            compare(out[b, h], lse[b, h], o_ref, l_ref, f"b{b} h{h}")


def test_bitmap_forward_8192_sampled():
    L = S = 8192
    q, k, v = W.random_qkv(1, 4, L, S, 64, torch.bfloat16, seed=31)
    words = W.random_bitmap(L, S, seed=32, p_empty=0.6, p_full=0.2)
    out, lse = run_gpu(q, k, v, OM.BITMAP, bitmap=words)
    rows = sample_rows(L, seed=6)
    for h in (0, 3):
        o_ref, l_ref = oracle_rows(q, k, v, 0, h, rows, OM.BITMAP, bitmap=words)
        compare(out[0, h][rows], lse[0, h][rows], o_ref, l_ref, f"h{h}")


def test_bitmap_of_causal_equals_causal_bit_for_bit():
    """The same keys are masked to -inf either way, so the outputs are identical."""
    L = S = 8192
    q, k, v = W.random_qkv(1, 8, L, S, 64, torch.bfloat16, seed=33)
    words = OM.to_bitmap(OM.CAUSAL, L, S, words_per_row=4 * (S // 128))
    ob, lb = run_gpu(q, k, v, OM.BITMAP, bitmap=words)
    oc, lc = run_gpu(q, k, v, OM.CAUSAL)
    assert torch.equal(ob, oc) and torch.equal(lb, lc)


def test_bitmap_empty_rows_and_all_ones():
    """A row with no bit set returns 0 / -inf; an all-ones bitmap is unmasked attention."""
    L, S = 400, 300
    q, k, v = W.random_qkv(1, 2, L, S, 64, torch.bfloat16, seed=34)
    words = W.random_bitmap(L, S, seed=35)
    words[17] = 0
    words[250:260] = 0
    out, lse = run_gpu(q, k, v, OM.BITMAP, bitmap=words)
    for r in [17] + list(range(250, 260)):
        assert torch.all(out[:, :, r] == 0) and torch.all(torch.isneginf(lse[:, :, r]))
    ones = OM.to_bitmap(OM.CAUSAL, L, S, words_per_row=4 * 3)
    ones[:] = np.uint32(0xFFFFFFFF)
    out, lse = run_gpu(q, k, v, OM.BITMAP, bitmap=ones)
    for h in range(2):
        o_ref, l_ref = oracle_rows(q, k, v, 0, h, np.arange(L), OM.BITMAP, bitmap=ones)
        compare(out[0, h], lse[0, h], o_ref, l_ref, f"h{h}")
