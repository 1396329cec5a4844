"""Decode against a KV cache on the GPU (split-KV tensor-core kernel + merge), against the fp64
CPU oracle: the lower-right causal, sliding-window and unmasked cases, grouped
query heads, softcap, ragged cache lengths, and rows that see no key."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention as OA
from oracle import masks as OM
from parity import compare

pytestmark = pytest.mark.gpu

# decode mask of the C-ABI -> oracle kind
ORACLE_KIND = {0: OM.DECODE_FULL, 1: OM.DECODE_CAUSAL, 2: OM.DECODE_SLIDING_WINDOW}


def _run(q, k, v, mask, window=0, sk=0, cap=0.0, scale=0.0):
    import block_sparse_attention_create_b200 as fa
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    out, lse = fa.flex_attention_decode(qd, kd, vd, mask=mask, window=window, score_mod=sk,
                                        softcap=cap, scale=scale, return_lse=True)
    torch.cuda.synchronize()
    assert fa.last_decode_error() == fa.FA_OK
    return out.cpu(), lse.cpu()


def _check(q, k, v, mask, window=0, sk=0, cap=0.0, scale=0.0, heads=None):
    out, lse = _run(q, k, v, mask, window, sk, cap, scale)
    B, H, L = q.shape[0], q.shape[1], q.shape[2]
    Hkv = k.shape[1]
    heads = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for (b, h) in heads:
        g = OA.kv_head(h, H, Hkv)
        o_ref, l_ref = OA.attention_head(q[b, h], k[b, g], v[b, g], ORACLE_KIND[mask],
                                         window=window or None, score_kind=sk, softcap=cap,
                                         scale=scale if scale > 0 else None)
        compare(out[b, h], lse[b, h], o_ref, l_ref, f"b{b} h{h}")
    return out, lse


@pytest.mark.parametrize("B,H,Hkv,L,S,D,mask,window", [
    (2, 8, 2, 1, 1000, 64, 1, 0), (1, 4, 4, 5, 3000, 128, 2, 300), (2, 4, 1, 3, 777, 64, 0, 0),
    (1, 8, 2, 4, 4099, 128, 1, 0), (3, 2, 2, 1, 64, 64, 1, 0), (1, 2, 1, 16, 129, 128, 2, 50)])
def test_decode_parity(B, H, Hkv, L, S, D, mask, window):
    q, k, v = W.random_qkv(B, H, L, S, D, torch.bfloat16, seed=B * 100 + S, Hkv=Hkv)
    _check(q, k, v, mask, window)


def test_decode_fp16_softcap_and_scale():
    q, k, v = W.random_qkv(1, 4, 2, 2000, 128, torch.float16, seed=51, scale=2.0, Hkv=2)
    _check(q, k, v, 1, sk=1, cap=30.0)
    _check(q, k, v, 2, window=700, scale=0.2)


def test_decode_long_cache_sampled_heads():
    """32 query heads over 8 K/V heads, one new token, 32768 cached keys."""
    q, k, v = W.random_qkv(1, 32, 1, 32768, 128, torch.bfloat16, seed=52, Hkv=8)
    _check(q, k, v, 1, heads=[(0, 0), (0, 13), (0, 31)])


def test_decode_rows_before_the_cache_see_nothing():
    """L > S: queries at negative key positions see no key (out 0, LSE -inf)."""
    q, k, v = W.random_qkv(1, 2, 8, 5, 64, torch.bfloat16, seed=53)
    out, lse = _check(q, k, v, 1)
    assert torch.all(out[:, :, :3] == 0) and torch.all(torch.isneginf(lse[:, :, :3]))


def test_decode_long_cache_32_rows_sampled_heads():
    """8 new tokens for 32 query heads over 8 K/V heads (32 rows per K/V head, two
    CTAs per chunk), 32768 cached keys."""
    q, k, v = W.random_qkv(1, 32, 8, 32768, 128, torch.bfloat16, seed=53, Hkv=8)
    _check(q, k, v, 1, heads=[(0, 0), (0, 5), (0, 31)])


def test_decode_window_skips_far_chunks_and_matches():
    """A small window over a long cache: most chunks load nothing."""
    q, k, v = W.random_qkv(2, 8, 1, 20000, 64, torch.bfloat16, seed=54, Hkv=8)
    _check(q, k, v, 2, window=100)


@pytest.mark.parametrize("B,H,Hkv,L,S,D,mask,window,dtype,xs", [
    (1, 3, 3, 1, 1000, 128, 1, 0, torch.bfloat16, 1.0),     # one row per K/V head
    (2, 6, 2, 1, 999, 64, 0, 0, torch.bfloat16, 1.0),       # three rows, ragged tail
    (1, 2, 1, 2, 4097, 128, 2, 500, torch.float16, 1.0),    # four rows, window
    (1, 1, 1, 4, 3, 64, 1, 0, torch.bfloat16, 1.0),         # L > S: a row sees nothing
    (1, 8, 2, 1, 6000, 128, 1, 0, torch.bfloat16, 2.0),     # x2 inputs: peaked rows
    (1, 8, 1, 1, 2500, 64, 1, 0, torch.bfloat16, 1.0),      # eight rows (the MMA's N)
    (2, 6, 2, 2, 1500, 128, 2, 400, torch.float16, 1.0),    # six rows, window
    (1, 4, 1, 1, 1000, 64, 0, 0, torch.float16, 2.0),       # fp16 at D = 64, no mask
    (1, 2, 2, 3, 0, 64, 1, 0, torch.bfloat16, 1.0),         # empty cache: no key at all
    (1, 3, 1, 3, 2049, 64, 1, 0, torch.bfloat16, 1.0),      # nine rows: a second row tile
    (1, 8, 1, 2, 3000, 128, 1, 0, torch.bfloat16, 2.0),     # sixteen rows, x2 inputs
    (2, 4, 1, 3, 1700, 64, 2, 350, torch.float16, 1.0),     # twelve rows, window, fp16
    (1, 4, 1, 4, 2, 128, 1, 0, torch.bfloat16, 1.0),        # sixteen rows, L > S
    (1, 8, 1, 3, 2500, 128, 1, 0, torch.bfloat16, 1.0),     # 24 rows: CTAs of 16 and 8 rows
    (1, 4, 1, 8, 1800, 64, 2, 300, torch.float16, 1.0),     # 32 rows, window
    (1, 1, 1, 17, 900, 64, 1, 0, torch.bfloat16, 1.0),      # 17 rows: a CTA with one row
])
def test_decode_tensor_core_path(B, H, Hkv, L, S, D, mask, window, dtype, xs):
    """Every decode runs on the warp-level tensor-core kernel: one or two 8-row column
    tiles, and a CTA per 16 rows beyond 16 (16-bit P against each warp's exact
    running max): element by element against the oracle."""
    q, k, v = W.random_qkv(B, H, L, S, D, dtype, seed=B * 1000 + S + L, scale=xs, Hkv=Hkv)
    out, lse = _check(q, k, v, mask, window)
    if L > S:
        assert torch.all(out[:, :, :L - S] == 0) and torch.all(torch.isneginf(lse[:, :, :L - S]))
