"""Pins for the CPU oracle: each test ties it to something other than itself.

Pins: the page-1 density table (golden), closed forms of the block counts,
brute-force loops on tiny shapes, torch's CPU SDPA in fp64 (a different
library routine), closed-form outputs (one visible key, all-equal scores,
a two-key softcap case), the tiled recurrence, and degenerate cases.
"""
import math

import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention as OA
from oracle import blockmask as OB
from oracle import bruteforce as BF
from oracle import masks as OM
from oracle import online as OO


def _rand(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape) * scale


# ---------------------------------------------------------------- block tables

def test_page1_density_table(golden):
    """Token and block densities printed on page 1 (results table)."""
    for pattern, seq, window, tok_pct, blk_pct in golden("page1_density_table.txt"):
        L = int(seq)
        if pattern == "causal":
            tok, blk = OB.densities(OM.CAUSAL, L, L)
        else:
            tok, blk = OB.densities(OM.SLIDING_WINDOW_CAUSAL, L, L, window=int(window))
        assert f"{100 * tok:.2f}" == tok_pct, (pattern, seq, window, tok)
        assert f"{100 * blk:.2f}" == blk_pct, (pattern, seq, window, blk)


@pytest.mark.parametrize("nq", [1, 2, 5, 64])
def test_causal_block_counts_closed_form(nq):
    """L = S = 128 nq: nq(nq+1)/2 live blocks; the diagonal ones are the partial ones."""
    t = OB.block_tables(OM.CAUSAL, 128 * nq, 128 * nq)
    assert int(t["kv_num_blocks"].sum()) == nq
    assert int(t["full_kv_num_blocks"].sum()) == nq * (nq - 1) // 2
    for i in range(nq):
        assert t["kv_num_blocks"][i] == 1 and t["kv_indices"][i, 0] == i
        assert list(t["full_kv_indices"][i, :i]) == list(range(i))


@pytest.mark.parametrize("nq,w", [(64, 256), (64, 1024), (40, 128), (64, 64), (30, 100)])
def test_window_block_counts_closed_form(nq, w):
    """Row i covers keys (q - W, q]; for W a multiple of 128 that is W/128 full blocks
    below the diagonal block, the oldest of them cut by the window (partial);
    for W < 128 the diagonal block and the one before it, both partial."""
    t = OB.block_tables(OM.SLIDING_WINDOW_CAUSAL, 128 * nq, 128 * nq, window=w)
    for i in range(nq):
        if w % 128 == 0:
            nb = w // 128
            exp_partial = [j for j in (i - nb, i) if j >= 0]
            exp_full = list(range(max(0, i - nb + 1), i))
        elif w < 128:
            exp_partial = [j for j in (i - 1, i) if j >= 0]
            exp_full = []
        else:  # 128 < W < 256, not a multiple: keys back to q - W + 1 reach block i - 2
            exp_partial = [j for j in (i - 2, i - 1, i) if j >= 0]
            exp_full = []
        got_p = list(t["kv_indices"][i, : t["kv_num_blocks"][i]])
        got_f = list(t["full_kv_indices"][i, : t["full_kv_num_blocks"][i]])
        assert got_p == exp_partial, (i, got_p, exp_partial)
        assert got_f == exp_full, (i, got_f, exp_full)


def test_window_32k_total_live_blocks():
    """3 live blocks per row except the first two rows: 3 * 256 - 3 = 765 of 65536."""
    t = OB.block_tables(OM.SLIDING_WINDOW_CAUSAL, 32768, 32768, window=256)
    live = t["kv_num_blocks"].sum() + t["full_kv_num_blocks"].sum()
    assert live == 3 * 256 - 3
    assert t["full_kv_num_blocks"].sum() == 255


def test_block_tables_unused_entries_are_zero():
    t = OB.block_tables(OM.SLIDING_WINDOW_CAUSAL, 1000, 1000, window=200)
    for i in range(t["n_q_blocks"]):
        assert not t["kv_indices"][i, t["kv_num_blocks"][i]:].any()
        assert not t["full_kv_indices"][i, t["full_kv_num_blocks"][i]:].any()


@pytest.mark.parametrize("kind,L,S,w", [
    (OM.CAUSAL, 300, 300, None), (OM.CAUSAL, 130, 260, None), (OM.CAUSAL, 260, 129, None),
    (OM.SLIDING_WINDOW_CAUSAL, 385, 385, 70), (OM.SLIDING_WINDOW_CAUSAL, 256, 200, 150),
    (OM.DOCUMENT_CAUSAL, 384, 384, None), (OM.CAUSAL, 1, 1, None), (OM.CAUSAL, 5, 0, None)])
def test_block_classification_bruteforce(kind, L, S, w):
    """Vectorised classification equals a per-pair loop, including ragged tails."""
    doc = None
    if kind == OM.DOCUMENT_CAUSAL:
        rng = np.random.default_rng(5)
        doc = rng.integers(0, 3, size=max(L, S))   # unsorted ids on purpose
    live, full, _ = OB.classify(kind, L, S, w, doc)
    for i in range(live.shape[0]):
        for j in range(live.shape[1]):
            c = BF.classify_block(kind, i, j, L, S, w, doc)
            assert (c != "empty") == live[i, j], (i, j, c)
            assert (c == "full") == full[i, j], (i, j, c)


# ---------------------------------------------------------------- attention

def _oracle(q, k, v, kind, **kw):
    return OA.attention_head(q, k, v, kind, **kw)


@pytest.mark.parametrize("L,S,D", [(1, 1, 64), (7, 7, 64), (128, 128, 64), (129, 129, 64),
                                   (200, 256, 64), (256, 200, 64), (33, 40, 128)])
@pytest.mark.parametrize("kind", [OM.CAUSAL, OM.SLIDING_WINDOW_CAUSAL, OM.DOCUMENT_CAUSAL])
def test_attention_bruteforce_tiny(L, S, D, kind):
    """Vectorised fp64 oracle equals pure-Python loops (scores, mask, softmax, LSE)."""
    if L * S * D > 256 * 200 * 64 // 2 and kind != OM.CAUSAL:
        pytest.skip("keep the pure-Python loops short")
    q, k, v = _rand((L, D), 1), _rand((S, D), 2), _rand((S, D), 3)
    w = 37 if kind == OM.SLIDING_WINDOW_CAUSAL else None
    doc = None
    if kind == OM.DOCUMENT_CAUSAL:
        doc = np.sort(np.random.default_rng(4).integers(0, 4, size=max(L, S)))
    sk = 1 if L % 2 else 0
    out, lse = _oracle(q, k, v, kind, window=w, doc_id=doc, score_kind=sk, softcap=3.0)
    bo, bl = BF.attention_head(q.tolist(), k.tolist(), v.tolist(), kind, w,
                               None if doc is None else doc.tolist(), sk, 3.0)
    np.testing.assert_allclose(out, np.array(bo).reshape(out.shape), rtol=0, atol=1e-12)
    bl = np.array(bl)
    assert np.array_equal(np.isinf(lse), np.isinf(bl))
    fin = np.isfinite(bl)
    np.testing.assert_allclose(lse[fin], bl[fin], rtol=0, atol=1e-12)


def test_rows_of_p_sum_to_one():
    """With V = 1 every live row's output is sum_j P_ij = 1 (up to the rounding
    of a sum of at most 300 fp64 terms, 300 * 2**-53 < 4e-14)."""
    L = 300
    q, k = _rand((L, 64), 10), _rand((L, 64), 11)
    v = np.ones((L, 64))
    for kind, w in ((OM.CAUSAL, None), (OM.SLIDING_WINDOW_CAUSAL, 50)):
        out, _ = _oracle(q, k, v, kind, window=w)
        assert np.abs(out - 1.0).max() <= 4e-14


def test_single_visible_key_returns_its_value():
    """Query 0 under every causal rule, and the first token of each document,
    see exactly one key: the output is that key's V, bit for bit."""
    L = 6000
    q, k, v = _rand((L, 64), 20), _rand((L, 64), 21), _rand((L, 64), 22)
    rows = np.array([0, 2048, 5000])
    doc = W.doc_id_from_starts(L, [2048, 5000]).numpy()
    out, lse = _oracle(q, k, v, OM.DOCUMENT_CAUSAL, doc_id=doc, rows=rows)
    for r, o in zip(rows, out):
        assert np.array_equal(o, v[r])
    for kind, w in ((OM.CAUSAL, None), (OM.SLIDING_WINDOW_CAUSAL, 256)):
        out, lse = _oracle(q, k, v, kind, window=w, rows=np.array([0]))
        assert np.array_equal(out[0], v[0])
        assert lse[0] == pytest.approx(float(q[0] @ k[0]) / 8.0, abs=1e-13)


def test_equal_scores_closed_form():
    """K = 0 makes every score 0: out is the mean of the visible V rows and
    lse = ln(number of visible keys), for each mask rule."""
    L = 700
    q, v = _rand((L, 64), 30), _rand((L, 64), 31)
    k = np.zeros((L, 64))
    starts = [0, 100, 333, 600]
    doc = W.doc_id_from_starts(L, starts[1:]).numpy()
    csum = np.cumsum(v, axis=0)
    for kind, w in ((OM.CAUSAL, None), (OM.SLIDING_WINDOW_CAUSAL, 64), (OM.DOCUMENT_CAUSAL, None)):
        out, lse = _oracle(q, k, v, kind, window=w, doc_id=doc)
        for i in range(L):
            if kind == OM.CAUSAL:
                lo = 0
            elif kind == OM.SLIDING_WINDOW_CAUSAL:
                lo = max(0, i - w + 1)
            else:
                lo = max(s for s in starts if s <= i)
            n = i - lo + 1
            mean = (csum[i] - (csum[lo - 1] if lo > 0 else 0)) / n
            assert np.abs(out[i] - mean).max() <= 1e-13
            assert abs(lse[i] - math.log(n)) <= 1e-13


def test_softcap_two_key_closed_form():
    """One key with scaled score 15 ln 3 (capped by c=30 to exactly 15, since
    tanh(ln 3 / 2) = 1/2) and one key with score 0: the weights are
    e^15 : 1.  Capping the unscaled score, dropping c, or skipping the cap
    all give different weights."""
    D = 64
    scale = 1.0 / 8.0
    x = 15.0 * math.log(3.0)
    q = np.zeros((2, D)); q[1, 0] = 1.0
    k = np.zeros((2, D)); k[0, 0] = x / scale
    v = np.zeros((2, D)); v[0, 1] = 1.0; v[1, 2] = 1.0
    out, lse = _oracle(q, k, v, OM.CAUSAL, score_kind=1, softcap=30.0)
    w0 = math.exp(15.0) / (math.exp(15.0) + 1.0)
    assert out[1, 1] == pytest.approx(w0, abs=1e-14)
    assert out[1, 2] == pytest.approx(1.0 - w0, abs=1e-14)
    assert lse[1] == pytest.approx(math.log(math.exp(15.0) + 1.0), abs=1e-12)


def test_softcap_infinite_cap_is_identity():
    L = 257
    q, k, v = _rand((L, 64), 40, 2.0), _rand((L, 64), 41, 2.0), _rand((L, 64), 42)
    a, la = _oracle(q, k, v, OM.CAUSAL)
    b, lb = _oracle(q, k, v, OM.CAUSAL, score_kind=1, softcap=1e30)
    assert np.abs(a - b).max() <= 1e-12 and np.abs(la - lb).max() <= 1e-12


def test_special_case_reductions():
    """W >= S turns the window rule into causal; one document is causal."""
    L = 400
    q, k, v = _rand((L, 64), 50), _rand((L, 64), 51), _rand((L, 64), 52)
    c, lc = _oracle(q, k, v, OM.CAUSAL)
    w, lw = _oracle(q, k, v, OM.SLIDING_WINDOW_CAUSAL, window=L)
    d, ld = _oracle(q, k, v, OM.DOCUMENT_CAUSAL, doc_id=np.zeros(L, dtype=np.int64))
    assert np.array_equal(c, w) and np.array_equal(lc, lw)
    assert np.array_equal(c, d) and np.array_equal(lc, ld)
    tc = OB.block_tables(OM.CAUSAL, L, L)
    tw = OB.block_tables(OM.SLIDING_WINDOW_CAUSAL, L, L, window=10 ** 6)
    for key in ("kv_num_blocks", "kv_indices", "full_kv_num_blocks", "full_kv_indices"):
        assert np.array_equal(tc[key], tw[key])


def test_fully_masked_rows_give_zero_and_minus_inf():
    """Window rule with L > S + W - 1: rows q >= S + W - 1 see no key."""
    L, S, w = 300, 100, 50
    q, k, v = _rand((L, 64), 60), _rand((S, 64), 61), _rand((S, 64), 62)
    out, lse = _oracle(q, k, v, OM.SLIDING_WINDOW_CAUSAL, window=w)
    dead = np.arange(L) >= S + w - 1
    assert np.all(out[dead] == 0.0) and np.all(np.isneginf(lse[dead]))
    assert np.all(np.isfinite(lse[~dead]))
    out0, lse0 = _oracle(q, k[:0], v[:0], OM.CAUSAL)
    assert np.all(out0 == 0.0) and np.all(np.isneginf(lse0))


@pytest.mark.parametrize("kind,w", [(OM.CAUSAL, None), (OM.SLIDING_WINDOW_CAUSAL, 100),
                                    (OM.DOCUMENT_CAUSAL, None)])
def test_matches_torch_sdpa_fp64(golden, kind, w):
    """torch's CPU SDPA in float64 given the same boolean mask (True = use the
    pair) agrees with the oracle to fp64 rounding; the SDPA tutorial's section 1
    measured SDPA against a naive implementation at 7.22e-16 / 1.11e-15 (golden)."""
    bound = max(float(r[2]) for r in golden("sdpa_fp64_equivalence.txt"))
    g = torch.Generator().manual_seed(0)
    q, k, v = (torch.randn(2, 8, 512, 64, generator=g, dtype=torch.float64) for _ in range(3))
    L = 512
    doc = np.sort(np.random.default_rng(1).integers(0, 5, size=L))
    mask = torch.from_numpy(OM.mask_rows(kind, np.arange(L), L, w, doc))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask)
    worst = 0.0
    for b in range(2):
        for h in range(8):
            o, _ = _oracle(q[b, h], k[b, h], v[b, h], kind, window=w, doc_id=doc)
            worst = max(worst, float(np.abs(o - ref[b, h].numpy()).max()))
    assert worst <= 10 * bound, worst


def test_sdpa_fully_masked_row_is_zero():
    """SDPA returns 0 (not NaN) for an all-False mask row (SDPA tutorial
    section 4); the oracle's reading for such rows agrees."""
    g = torch.Generator().manual_seed(3)
    q, k, v = (torch.randn(1, 1, 4, 8, generator=g, dtype=torch.float64) for _ in range(3))
    mask = torch.zeros(1, 1, 4, 4, dtype=torch.bool)
    mask[..., 1:, 0] = True
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask)
    assert torch.all(ref[0, 0, 0] == 0)
    # oracle with window 1 and S shifted: row 0 of a window rule over keys 1.. sees nothing
    out, lse = _oracle(q[0, 0].numpy(), k[0, 0, :0].numpy(), v[0, 0, :0].numpy(), OM.CAUSAL)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


# ---------------------------------------------------------------- tiled recurrence

def test_tiled_softmax_matches_plain(golden):
    """Running-max softmax over 4096 values vs plain softmax (page 3 table)."""
    x = _rand((4096,), 70)     # N(0,1): softmax entries ~1/4096, as on the page
    plain = np.exp(x - x.max()) / np.exp(x - x.max()).sum()
    for tile, max_err, _ in golden("tiled_softmax_errors.txt"):
        got = OO.softmax_tiled_1d(x, int(tile))
        err = np.abs(got - plain).max()
        assert err < 1e-9          # the page's acceptance threshold
        assert err <= 100 * float(max_err) + 1e-17


@pytest.mark.parametrize("kind,w,sk", [(OM.CAUSAL, None, 0), (OM.SLIDING_WINDOW_CAUSAL, 300, 1),
                                       (OM.DOCUMENT_CAUSAL, None, 0)])
def test_tiled_attention_matches_dense(kind, w, sk):
    L = 1000
    q, k, v = _rand((L, 64), 80), _rand((L, 64), 81), _rand((L, 64), 82)
    doc = W.doc_id_from_starts(L, [200, 640]).numpy()
    a, la = OA.attention_head(q, k, v, kind, window=w, doc_id=doc, score_kind=sk, softcap=5.0)
    b, lb = OO.attention_head_tiled(q, k, v, kind, window=w, doc_id=doc, score_kind=sk, softcap=5.0)
    assert np.abs(a - b).max() <= 1e-14
    assert np.abs(la - lb).max() <= 1e-13


def test_row_subset_equals_full():
    L = 600
    q, k, v = _rand((L, 64), 90), _rand((L, 64), 91), _rand((L, 64), 92)
    full, lf = OA.attention_head(q, k, v, OM.CAUSAL)
    rows = np.array([5, 599, 128, 0, 300])
    sub, ls = OA.attention_head(q, k, v, OM.CAUSAL, rows=rows)
    # BLAS may block a different row set differently: equal up to fp64 rounding
    assert np.abs(full[rows] - sub).max() <= 1e-14 and np.abs(lf[rows] - ls).max() <= 1e-13


def test_workload_generators_are_seeded():
    a = W.make_qkv(W.C1_CAUSAL_256)
    b = W.make_qkv(W.C1_CAUSAL_256)
    for x, y in zip(a, b):
        assert torch.equal(x, y) and x.dtype == torch.bfloat16
    d = W.make_doc_id(W.C4_DOC_SEEDED)
    n_docs = int(d.max()) + 1
    assert 4 <= n_docs <= 16 and d.shape == (8192,)
    assert torch.all(d[1:] >= d[:-1])
    f = W.make_doc_id(W.C4_DOC_FIXED)
    assert int(f[2047]) == 0 and int(f[2048]) == 1 and int(f[4999]) == 1 and int(f[5000]) == 2


# ---------------------------------------------------------------- tabulated mask_mod

def test_bitmap_layout_hand_example():
    """Causal 3 x 3 tabulated by hand: row q keeps keys 0..q, bit kv of word 0."""
    words = OM.to_bitmap(OM.CAUSAL, 3, 3)
    assert words.tolist() == [[0b1], [0b11], [0b111]]
    # key 33 of row 0 lives in word 1, bit 1
    w = np.zeros((1, 2), dtype=np.uint32)
    w[0, 1] = 2
    assert OM.mask_rows(OM.BITMAP, [0], 64, bitmap=w).nonzero()[1].tolist() == [33]


@pytest.mark.parametrize("kind,L,S,w", [
    (OM.CAUSAL, 300, 300, None), (OM.CAUSAL, 1000, 300, None), (OM.CAUSAL, 200, 700, None),
    (OM.SLIDING_WINDOW_CAUSAL, 385, 385, 70), (OM.DOCUMENT_CAUSAL, 384, 384, None)])
def test_bitmap_of_a_rule_reduces_to_the_rule(kind, L, S, w):
    """A bitmap tabulating a mask rule gives that rule's block tables and outputs."""
    doc = None
    if kind == OM.DOCUMENT_CAUSAL:
        doc = np.random.default_rng(7).integers(0, 3, size=max(L, S))
    words = OM.to_bitmap(kind, L, S, w, doc, words_per_row=4 * (-(-S // 128)))
    a = OB.block_tables(kind, L, S, w, doc)
    b = OB.block_tables(OM.BITMAP, L, S, bitmap=words)
    for key in ("kv_num_blocks", "kv_indices", "full_kv_num_blocks", "full_kv_indices"):
        assert np.array_equal(a[key], b[key]), key
    q, k, v = (_rand((n, 32), s) for n, s in ((L, 1), (S, 2), (S, 3)))
    oa, la = OA.attention_head(q, k, v, kind, window=w, doc_id=doc)
    ob, lb = OA.attention_head(q, k, v, OM.BITMAP, bitmap=words)
    assert np.array_equal(oa, ob) and np.array_equal(la, lb)


@pytest.mark.parametrize("L,S", [(7, 9), (130, 70), (64, 200)])
def test_bitmap_bruteforce_tiny(L, S):
    """Vectorised oracle on a random bitmap equals pure-Python loops."""
    words = W.random_bitmap(L, S, seed=L + S)
    q, k, v = (_rand((n, 16), s) for n, s in ((L, 4), (S, 5), (S, 6)))
    out, lse = OA.attention_head(q, k, v, OM.BITMAP, bitmap=words)
    bo, bl = BF.attention_head(q.tolist(), k.tolist(), v.tolist(), OM.BITMAP, bitmap=words)
    assert np.allclose(out, np.array(bo), atol=1e-12, rtol=0)
    assert np.allclose(lse, np.array(bl), atol=1e-12, rtol=0, equal_nan=False)
    live, full, _ = OB.classify(OM.BITMAP, L, S, bitmap=words)
    for i in range(live.shape[0]):
        for j in range(live.shape[1]):
            c = BF.classify_block(OM.BITMAP, i, j, L, S, bitmap=words)
            assert (c != "empty") == live[i, j] and (c == "full") == full[i, j], (i, j, c)


def test_bitmap_matches_torch_sdpa_fp64():
    """torch's CPU SDPA in fp64 given the bitmap as a boolean mask built by
    per-pair bit extraction."""
    L = S = 300
    words = W.random_bitmap(L, S, seed=9)
    mask = torch.tensor([[(int(words[qq][kk // 32]) >> (kk % 32)) & 1 == 1 for kk in range(S)]
                         for qq in range(L)])
    live_rows = mask.any(dim=1)
    q, k, v = (torch.from_numpy(_rand((1, 1, n, 32), s)) for n, s in ((L, 1), (S, 2), (S, 3)))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask)[0, 0].numpy()
    out, lse = OA.attention_head(q[0, 0], k[0, 0], v[0, 0], OM.BITMAP, bitmap=words)
    assert np.abs(out[live_rows.numpy()] - ref[live_rows.numpy()]).max() < 1e-12
    assert np.all(out[~live_rows.numpy()] == 0) and np.all(np.isneginf(lse[~live_rows.numpy()]))


@pytest.mark.parametrize("kind,L,S,w", [
    (OM.CAUSAL, 300, 300, None), (OM.SLIDING_WINDOW_CAUSAL, 700, 500, 200),
    (OM.DOCUMENT_CAUSAL, 384, 384, None), (OM.BITMAP, 400, 300, None)])
def test_transpose_matches_bruteforce(kind, L, S, w):
    """Column lists (q blocks per kv block, ascending) from per-pair classification."""
    doc = np.random.default_rng(3).integers(0, 3, size=max(L, S)) if kind == OM.DOCUMENT_CAUSAL \
        else None
    words = W.random_bitmap(L, S, seed=11) if kind == OM.BITMAP else None
    t = OB.transpose(OB.block_tables(kind, L, S, w, doc, bitmap=words))
    nq, nkv = -(-L // 128), -(-S // 128)
    for j in range(nkv):
        cls = [BF.classify_block(kind, i, j, L, S, w, doc, bitmap=words) for i in range(nq)]
        part = [i for i in range(nq) if cls[i] == "partial"]
        full = [i for i in range(nq) if cls[i] == "full"]
        assert t["q_num_blocks"][j] == len(part) and t["full_q_num_blocks"][j] == len(full)
        assert t["q_indices"][j].tolist() == part + [0] * (nq - len(part))
        assert t["full_q_indices"][j].tolist() == full + [0] * (nq - len(full))


# ---------------------------------------------------------------- grouped-query attention

@pytest.mark.parametrize("H,Hkv", [(8, 2), (4, 1), (6, 6)])
def test_gqa_matches_torch_sdpa_enable_gqa(H, Hkv):
    """Batched oracle with H query heads over Hkv K/V heads equals torch's CPU SDPA
    in fp64 with enable_gqa=True (its own head grouping), causal and window."""
    B, L = 2, 200
    q = torch.from_numpy(_rand((B, H, L, 32), 1))
    k = torch.from_numpy(_rand((B, Hkv, L, 32), 2))
    v = torch.from_numpy(_rand((B, Hkv, L, 32), 3))
    for kind, w in ((OM.CAUSAL, None), (OM.SLIDING_WINDOW_CAUSAL, 50)):
        mask = torch.from_numpy(OM.mask_rows(kind, np.arange(L), L, w))
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask,
                                                               enable_gqa=True).numpy()
        res = OA.attention(q, k, v, kind, window=w)
        for (b, h), (out, _) in res.items():
            assert np.abs(out - ref[b, h]).max() < 1e-12, (b, h)


def test_gqa_head_map_hand_example():
    """32 query heads over 8 K/V heads: heads 0-3 -> 0, 4-7 -> 1, ..., 28-31 -> 7."""
    assert [OA.kv_head(h, 32, 8) for h in range(32)] == [h // 4 for h in range(32)]
    assert [OA.kv_head(h, 5, 1) for h in range(5)] == [0] * 5
    with pytest.raises(ValueError):
        OA.kv_head(0, 6, 4)


# ---------------------------------------------------------------- decode (KV cache)

@pytest.mark.parametrize("L,S", [(1, 6), (1, 300), (5, 300), (64, 1000)])
def test_decode_rows_equal_last_rows_of_full_causal(L, S):
    """SDPA tutorial, section 4, pitfall 3: decoding the last L queries against the
    whole cache with the lower-right causal mask equals the last L rows of causal
    attention over all S queries (L = S, where both alignments agree)."""
    q_all, k, v = _rand((S, 32), 1), _rand((S, 32), 2), _rand((S, 32), 3)
    full, lfull = OA.attention_head(q_all, k, v, OM.CAUSAL, rows=np.arange(S - L, S))
    dec, ldec = OA.attention_head(q_all[S - L:], k, v, OM.DECODE_CAUSAL)
    assert np.array_equal(full, dec) and np.array_equal(lfull, ldec)
    fw, lw = OA.attention_head(q_all, k, v, OM.SLIDING_WINDOW_CAUSAL, window=40,
                               rows=np.arange(S - L, S))
    dw, ldw = OA.attention_head(q_all[S - L:], k, v, OM.DECODE_SLIDING_WINDOW, window=40)
    assert np.array_equal(fw, dw) and np.array_equal(lw, ldw)


def test_decode_matches_torch_causal_lower_right():
    """torch's CPU SDPA in fp64 with its causal_lower_right bias."""
    from torch.nn.attention.bias import causal_lower_right
    L, S = 7, 200
    q = torch.from_numpy(_rand((1, 2, L, 32), 4))
    k = torch.from_numpy(_rand((1, 2, S, 32), 5))
    v = torch.from_numpy(_rand((1, 2, S, 32), 6))
    ref = torch.nn.functional.scaled_dot_product_attention(
        q, k, v, attn_mask=causal_lower_right(L, S)).numpy()
    nomask = torch.nn.functional.scaled_dot_product_attention(q, k, v).numpy()
    for h in range(2):
        out, _ = OA.attention_head(q[0, h], k[0, h], v[0, h], OM.DECODE_CAUSAL)
        assert np.abs(out - ref[0, h]).max() < 1e-12
        full, _ = OA.attention_head(q[0, h], k[0, h], v[0, h], OM.DECODE_FULL)
        assert np.abs(full - nomask[0, h]).max() < 1e-12


@pytest.mark.parametrize("kind", [OM.DECODE_FULL, OM.DECODE_CAUSAL, OM.DECODE_SLIDING_WINDOW])
def test_decode_bruteforce_tiny(kind):
    L, S = 3, 11
    q, k, v = (_rand((n, 8), s) for n, s in ((L, 7), (S, 8), (S, 9)))
    out, lse = OA.attention_head(q, k, v, kind, window=4)
    bo, bl = BF.attention_head(q.tolist(), k.tolist(), v.tolist(), kind, 4)
    assert np.allclose(out, np.array(bo), atol=1e-13, rtol=0)
    assert np.allclose(lse, np.array(bl), atol=1e-13, rtol=0)


# ---------------------------------------------------------------- backward

from oracle import backward as OBW  # noqa: E402


@pytest.mark.parametrize("kind,w", [(OM.CAUSAL, None), (OM.SLIDING_WINDOW_CAUSAL, 40),
                                    (OM.DOCUMENT_CAUSAL, None), (OM.BITMAP, None)])
def test_backward_matches_torch_autograd_fp64(kind, w):
    """Gradients equal torch autograd through its CPU SDPA in fp64 with the same
    boolean mask (rows with no live key excluded from SDPA's comparison)."""
    L, S, D = 150, 130, 16
    doc = np.random.default_rng(2).integers(0, 3, size=max(L, S)) if kind == OM.DOCUMENT_CAUSAL \
        else None
    words = W.random_bitmap(L, S, seed=3) if kind == OM.BITMAP else None
    mask = OM.mask_rows(kind, np.arange(L), S, w, doc, words, q_len=L)
    live = mask.any(axis=1)
    q, k, v, do = (_rand(shape, s) for shape, s in (((L, D), 1), ((S, D), 2), ((S, D), 3),
                                                    ((L, D), 4)))
    do[~live] = 0.0   # SDPA gives dead rows a zero output; give them no gradient either
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(tq[None, None], tk[None, None],
                                                           tv[None, None],
                                                           attn_mask=torch.from_numpy(mask))
    out[0, 0].backward(torch.from_numpy(do))
    dq, dk, dv = OBW.attention_head_backward(q, k, v, do, kind, window=w, doc_id=doc, bitmap=words)
    assert np.abs(dq - tq.grad.numpy()).max() < 1e-10
    assert np.abs(dk - tk.grad.numpy()).max() < 1e-10
    assert np.abs(dv - tv.grad.numpy()).max() < 1e-10


def test_backward_softcap_finite_differences():
    """Central differences of sum(out * dO) reproduce every gradient under the softcap."""
    L, S, D = 5, 7, 4
    q, k, v, do = (_rand(shape, s, 2.0) for shape, s in (((L, D), 5), ((S, D), 6), ((S, D), 7),
                                                         ((L, D), 8)))
    args = dict(score_kind=1, softcap=1.5)

    def f(qq, kk, vv):
        out, _ = OA.attention_head(qq, kk, vv, OM.SLIDING_WINDOW_CAUSAL, window=4, **args)
        return float((out * do).sum())
    dq, dk, dv = OBW.attention_head_backward(q, k, v, do, OM.SLIDING_WINDOW_CAUSAL, window=4, **args)
    h = 1e-6
    for x, g, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            a = [q, k, v]
            a[which] = xp
            fp = f(*a)
            a[which] = xm
            fm = f(*a)
            assert abs((fp - fm) / (2 * h) - g[idx]) < 1e-7, (which, idx)


def test_backward_single_visible_key_closed_form():
    """Causal row 0 sees key 0 alone: P = 1 there, so dO_0 . v_0 equals the row sum
    rowsum(dO_0 * O_0) and dS vanishes on the row, giving dq_0 = 0; its only effect on
    dv is dO_0 added to dv_0, and it adds nothing to dk."""
    L, S, D = 6, 6, 8
    q, k, v, do = (_rand((n, D), s) for n, s in ((L, 11), (S, 12), (S, 13), (L, 14)))
    dq, dk, dv = OBW.attention_head_backward(q, k, v, do, OM.CAUSAL)
    assert np.abs(dq[0]).max() < 1e-12
    do_rest = do.copy()
    do_rest[0] = 0.0
    _, dk_rest, dv_rest = OBW.attention_head_backward(q, k, v, do_rest, OM.CAUSAL)
    assert np.abs(dv[0] - dv_rest[0] - do[0]).max() < 1e-12
    assert np.abs(dv[1:] - dv_rest[1:]).max() < 1e-12
    assert np.abs(dk - dk_rest).max() < 1e-12


def test_backward_grouped_heads_sum_over_the_group():
    """With two query heads on one K/V head, dk and dv of the shared head are the
    sums of the per-head gradients: checked against torch autograd through fp64
    SDPA with enable_gqa."""
    L, S, D = 40, 40, 8
    q = np.stack([_rand((L, D), 21), _rand((L, D), 22)])
    k, v = _rand((S, D), 23), _rand((S, D), 24)
    do = np.stack([_rand((L, D), 25), _rand((L, D), 26)])
    mask = OM.mask_rows(OM.SLIDING_WINDOW_CAUSAL, np.arange(L), S, 9, q_len=L)
    tq = torch.tensor(q[None], requires_grad=True)
    tk = torch.tensor(k[None, None], requires_grad=True)
    tv = torch.tensor(v[None, None], requires_grad=True)
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv,
                                                           attn_mask=torch.from_numpy(mask),
                                                           enable_gqa=True)
    out.backward(torch.from_numpy(do[None]))
    dk = np.zeros((S, D))
    dv = np.zeros((S, D))
    for h in range(2):
        gq, gk, gv = OBW.attention_head_backward(q[h], k, v, do[h], OM.SLIDING_WINDOW_CAUSAL,
                                                 window=9)
        assert np.abs(gq - tq.grad.numpy()[0, h]).max() < 1e-10
        dk += gk
        dv += gv
    assert np.abs(dk - tk.grad.numpy()[0, 0]).max() < 1e-10
    assert np.abs(dv - tv.grad.numpy()[0, 0]).max() < 1e-10


@pytest.mark.parametrize("kind,w,sk", [(OM.CAUSAL, None, 0), (OM.SLIDING_WINDOW_CAUSAL, 37, 0),
                                       (OM.DOCUMENT_CAUSAL, None, 1), (OM.BITMAP, None, 0)])
def test_backward_sampled_rows_equal_the_dense_gradients(kind, w, sk):
    """The sampled form gives the dense form's rows of dq, dk, dv, P and dS, for
    scattered query and key samples (the dense form is pinned to torch autograd)."""
    L, S, D = 300, 260, 16
    doc = np.random.default_rng(5).integers(0, 4, size=max(L, S)) \
        if kind == OM.DOCUMENT_CAUSAL else None
    words = W.random_bitmap(L, S, seed=9) if kind == OM.BITMAP else None
    q, k, v, do = (_rand(shape, s) for shape, s in (((L, D), 31), ((S, D), 32), ((S, D), 33),
                                                    ((L, D), 34)))
    args = dict(window=w, doc_id=doc, bitmap=words, score_kind=sk, softcap=4.0 if sk else 0.0)
    dq, dk, dv, p, ds = OBW.attention_head_backward(q, k, v, do, kind, return_probs=True, **args)
    g = np.random.default_rng(7)
    q_rows = np.concatenate([[0, L - 1], g.choice(L, 20, replace=False)])
    k_rows = np.concatenate([[S - 1, 0], g.choice(S, 20, replace=False)])
    r = OBW.attention_head_backward_sampled(q, k, v, do, kind, q_rows, k_rows, chunk=64, **args)
    assert np.abs(r["dq"] - dq[q_rows]).max() < 1e-12
    assert np.abs(r["dk"] - dk[k_rows]).max() < 1e-12
    assert np.abs(r["dv"] - dv[k_rows]).max() < 1e-12
    assert np.abs(r["p"] - p[r["rows"]]).max() < 1e-13
    assert np.abs(r["ds"] - ds[r["rows"]]).max() < 1e-12
    # every row with a live pair on a sampled key was evaluated
    sees = OM.mask_rows(kind, np.arange(L), S, w, doc, words, q_len=L)[:, k_rows].any(axis=1)
    assert set(np.flatnonzero(sees)) <= set(r["rows"].tolist())
