"""Failure detection on the GPU without a fault: with the testing hook that makes
the forward kernel's MMA warp issue nothing, every bounded wait of the kernel runs
out, the kernel stops all roles and returns, the host reads FA_ERR_TIMEOUT from the
workspace error word, and the context stays usable for the next, correct call."""
import time

import numpy as np
import pytest
import torch

import workloads as W
from oracle import masks as OM
from parity import compare, oracle_rows

pytestmark = pytest.mark.gpu


def test_bounded_waits_report_timeout_and_context_survives():
    import block_sparse_attention_create_b200 as fa
    q, k, v = W.random_qkv(1, 2, 1000, 1000, 64, torch.bfloat16, seed=61)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    bm = fa.create_block_mask(OM.SLIDING_WINDOW_CAUSAL, 1000, 1000, window=300, device="cuda")
    torch.cuda.synchronize()
    assert fa.last_device_error() == fa.FA_OK          # start from a clear error word
    fa.fa_debug_set_mma_stall(1, 50_000_000)           # 50 ms wait limit
    try:
        t0 = time.perf_counter()
        fa.flex_attention(qd, kd, vd, bm)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        fa.fa_debug_set_mma_stall(0, 0)
    assert fa.last_device_error() == fa.FA_ERR_TIMEOUT
    assert elapsed < 10.0
    assert fa.last_device_error() == fa.FA_OK          # reading cleared it
    out, lse = fa.flex_attention(qd, kd, vd, bm, return_lse=True)
    torch.cuda.synchronize()
    assert fa.last_device_error() == fa.FA_OK
    rows = np.arange(0, 1000, 7)
    for h in range(2):
        o_ref, l_ref = oracle_rows(q, k, v, 0, h, rows, OM.SLIDING_WINDOW_CAUSAL, 300)
        compare(out[0, h].cpu()[rows], lse[0, h].cpu()[rows], o_ref, l_ref, f"h{h}")


def test_decode_bounded_waits_report_timeout_and_context_survives():
    """The decode kernel's waits on its K/V tiles are bounded too: with the hook on,
    no tile is loaded, every CTA's first wait runs out, the CTAs return, the host
    reads FA_ERR_TIMEOUT from the decode workspace, and the next decode is correct."""
    import block_sparse_attention_create_b200 as fa
    B, H, Hkv, L, S, D = 2, 8, 2, 1, 4096, 128
    g = torch.Generator().manual_seed(63)
    q = torch.randn(B, H, L, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B, Hkv, S, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, S, D, generator=g).to(torch.bfloat16)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    fa.flex_attention_decode(qd, kd, vd, mask=fa.FA_DECODE_CAUSAL)
    torch.cuda.synchronize()
    assert fa.last_decode_error() == fa.FA_OK
    fa.fa_debug_set_mma_stall(1, 50_000_000)
    try:
        t0 = time.perf_counter()
        fa.flex_attention_decode(qd, kd, vd, mask=fa.FA_DECODE_CAUSAL)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        fa.fa_debug_set_mma_stall(0, 0)
    assert fa.last_decode_error() == fa.FA_ERR_TIMEOUT
    assert elapsed < 10.0
    assert fa.last_decode_error() == fa.FA_OK
    out, lse = fa.flex_attention_decode(qd, kd, vd, mask=fa.FA_DECODE_CAUSAL, return_lse=True)
    torch.cuda.synchronize()
    assert fa.last_decode_error() == fa.FA_OK
    from oracle import attention as OA
    for b, h in ((0, 0), (1, 7)):
        o_ref, l_ref = OA.attention_head(q[b, h], k[b, h // (H // Hkv)], v[b, h // (H // Hkv)],
                                         OM.DECODE_CAUSAL)
        compare(out[b, h].cpu(), lse[b, h].cpu(), o_ref, l_ref, f"b{b} h{h}")


def test_backward_bounded_waits_report_timeout_and_context_survives():
    """The backward's tcgen05 kernels wait on bounded mbarriers as well: with the hook
    on, no tile is loaded, the waits run out, the error word reads FA_ERR_TIMEOUT,
    and the next backward on the same context is correct."""
    import block_sparse_attention_create_b200 as fa
    from oracle import backward as OB
    L = 300
    q, k, v = W.random_qkv(1, 2, L, L, 64, torch.bfloat16, seed=64)
    g = torch.Generator().manual_seed(65)
    do = torch.randn(1, 2, L, 64, generator=g).to(torch.bfloat16)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    bm = fa.create_block_mask(OM.CAUSAL, L, L, device="cuda")
    out, lse = fa.flex_attention(qd, kd, vd, bm, return_lse=True)
    torch.cuda.synchronize()
    fa.fa_debug_set_mma_stall(1, 50_000_000)
    try:
        with pytest.raises(fa.FAError) as err:
            fa.flex_attention_backward(qd, kd, vd, out, dod, lse, bm, check=True)
    finally:
        fa.fa_debug_set_mma_stall(0, 0)
    assert err.value.status == fa.FA_ERR_TIMEOUT
    dq, dk, dv = fa.flex_attention_backward(qd, kd, vd, out, dod, lse, bm, check=True)
    torch.cuda.synchronize()
    ref = OB.attention_head_backward(q[0, 1], k[0, 1], v[0, 1], do[0, 1], OM.CAUSAL)
    for got, want in zip((dq[0, 1], dk[0, 1], dv[0, 1]), ref):
        err_abs = (got.cpu().double() - torch.as_tensor(want)).abs().max().item()
        assert err_abs < 0.05 * (float(torch.as_tensor(want).abs().max()) + 1e-3) + 2e-2, err_abs
