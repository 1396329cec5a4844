"""Per-(batch, head) masks on the GPU (create_block_mask with B and / or H given):
each instance's block tables and column lists bit-exact against the oracle, the
forward of every (b, h) against the fp64 oracle with that instance's mask, and
identical instances giving the broadcast mask's output bit for bit."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import blockmask as OB
from oracle import masks as OM
from parity import compare, oracle_rows, run_gpu

pytestmark = pytest.mark.gpu

KEYS = ("kv_num_blocks", "kv_indices", "full_kv_num_blocks", "full_kv_indices")
T_KEYS = ("q_num_blocks", "q_indices", "full_q_num_blocks", "full_q_indices")


def _docs(n_inst, n, seed):
    g = torch.Generator().manual_seed(seed)
    out = []
    for _ in range(n_inst):  # sorted documents with random boundaries, different per instance
        cuts = sorted(int(c) for c in torch.randperm(n - 1, generator=g)[:3] + 1)
        out.append(W.doc_id_from_starts(n, cuts))
    return torch.stack(out).contiguous()


def _run_bh(q, k, v, kind, doc=None, words=None, mb=1, mh=1):
    import block_sparse_attention_create_b200 as fa
    L, S = q.shape[2], k.shape[2]
    bits = (torch.from_numpy(np.ascontiguousarray(words).view(np.int32)).cuda()
            if words is not None else None)
    bm = fa.create_block_mask(kind, L, S, doc_id=doc.cuda() if doc is not None else None,
                              bitmap=bits, B=mb, H=mh)
    out, lse = fa.flex_attention(q.cuda(), k.cuda(), v.cuda(), bm, return_lse=True)
    torch.cuda.synchronize()
    assert fa.last_device_error() == fa.FA_OK
    return bm, out.cpu(), lse.cpu()


def _inst(b, h, mb, mh):
    return (b if mb > 1 else 0) * mh + (h if mh > 1 else 0)


@pytest.mark.parametrize("B,H,mb,mh,L", [(3, 2, 3, 1, 1000), (2, 3, 2, 3, 700), (1, 4, 1, 4, 513)])
def test_per_instance_documents(B, H, mb, mh, L):
    q, k, v = W.random_qkv(B, H, L, L, 64, torch.bfloat16, seed=71 + L)
    doc = _docs(mb * mh, L, seed=L)
    bm, out, lse = _run_bh(q, k, v, OM.DOCUMENT_CAUSAL, doc=doc, mb=mb, mh=mh)
    got = bm.tables()
    t_got = {key: t.cpu().numpy() for key, t in bm.transpose().items()}
    nq, nkv = bm.n_q_blocks, bm.n_kv_blocks
    for n in range(mb * mh):
        ref = OB.block_tables(OM.DOCUMENT_CAUSAL, L, L, doc_id=doc[n].numpy())
        for key in KEYS:
            g = got[key].reshape(mb * mh, nq, -1)[n].reshape(ref[key].shape)
            assert np.array_equal(g, ref[key]), (n, key)
        tref = OB.transpose(ref)
        for key in T_KEYS:
            g = t_got[key].reshape(mb * mh, nkv, -1)[n].reshape(tref[key].shape)
            assert np.array_equal(g, tref[key]), (n, key)
    for b in range(B):
        for h in range(H):
            d = doc[_inst(b, h, mb, mh)]
            o_ref, l_ref = oracle_rows(q, k, v, b, h, np.arange(L), OM.DOCUMENT_CAUSAL, 0, d)
            compare(out[b, h], lse[b, h], o_ref, l_ref, f"b{b} h{h}")


def test_per_head_bitmaps_with_grouped_heads():
    """One tabulated mask per query head, 4 query heads sharing 2 K/V heads."""
    L, S, H = 400, 300, 4
    q, k, v = W.random_qkv(1, H, L, S, 128, torch.bfloat16, seed=81, Hkv=2)
    words = np.stack([W.random_bitmap(L, S, seed=90 + h) for h in range(H)])
    _, out, lse = _run_bh(q, k, v, OM.BITMAP, words=words, mh=H)
    for h in range(H):
        o_ref, l_ref = oracle_rows(q, k, v, 0, h, np.arange(L), OM.BITMAP, bitmap=words[h])
        compare(out[0, h], lse[0, h], o_ref, l_ref, f"h{h}")


def test_identical_instances_equal_broadcast_bit_for_bit():
    B, H, L = 2, 3, 1500
    q, k, v = W.random_qkv(B, H, L, L, 64, torch.float16, seed=82)
    one = _docs(1, L, seed=5)
    _, ob, lb = _run_bh(q, k, v, OM.DOCUMENT_CAUSAL, doc=one.repeat(B * H, 1), mb=B, mh=H)
    oc, lc = run_gpu(q, k, v, OM.DOCUMENT_CAUSAL, doc_id=one[0])
    assert torch.equal(ob, oc) and torch.equal(lb, lc)


@pytest.mark.parametrize("D", [64, 128])
def test_backward_per_instance_masks(D):
    """Backward with per-(batch, head) masks: documents per batch element and head,
    then per-head tabulated masks with grouped heads; every (b, h) against the fp64
    oracle's gradients with that instance's mask (dk / dv of a K/V head summed over
    its query heads)."""
    import block_sparse_attention_create_b200 as fa
    from oracle import backward as OBW

    def check(got, ref, what):
        got = got.double().numpy()
        rms = float(np.sqrt((ref ** 2).mean())) + 1e-6
        err = np.abs(got - ref)
        assert (err <= 3e-2 * (np.abs(ref) + rms) + 1e-3).all(), (what, float(err.max()))

    # documents per (b, h)
    B, H, L = 2, 2, 520
    q, k, v = W.random_qkv(B, H, L, L, D, torch.bfloat16, seed=91 + D)
    dout = torch.randn(B, H, L, D, generator=torch.Generator().manual_seed(92)).to(torch.bfloat16)
    doc = _docs(B * H, L, seed=93)
    bm = fa.create_block_mask(OM.DOCUMENT_CAUSAL, L, L, doc_id=doc.cuda(), B=B, H=H)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, dout))
    out, lse = fa.flex_attention(qd, kd, vd, bm, return_lse=True)
    dq, dk, dv = fa.flex_attention_backward(qd, kd, vd, out, dod, lse, bm, check=True)
    for b in range(B):
        for h in range(H):
            ref = OBW.attention_head_backward(q[b, h], k[b, h], v[b, h], dout[b, h],
                                              OM.DOCUMENT_CAUSAL, doc_id=doc[b * H + h].numpy())
            for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
                check(got[b, h].cpu(), want, f"doc b{b} h{h} {name}")
    # per-head bitmaps, 4 query heads over 2 K/V heads
    L, S, H, Hkv = 300, 260, 4, 2
    q, k, v = W.random_qkv(1, H, L, S, D, torch.bfloat16, seed=94 + D, Hkv=Hkv)
    dout = torch.randn(1, H, L, D, generator=torch.Generator().manual_seed(95)).to(torch.bfloat16)
    words = np.stack([W.random_bitmap(L, S, seed=96 + h) for h in range(H)])
    bits = torch.from_numpy(np.ascontiguousarray(words).view(np.int32)).cuda()
    bm = fa.create_block_mask(OM.BITMAP, L, S, bitmap=bits, H=H)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, dout))
    out, lse = fa.flex_attention(qd, kd, vd, bm, return_lse=True)
    dq, dk, dv = fa.flex_attention_backward(qd, kd, vd, out, dod, lse, bm, check=True)
    G = H // Hkv
    refs = [OBW.attention_head_backward(q[0, h], k[0, h // G], v[0, h // G], dout[0, h],
                                        OM.BITMAP, bitmap=words[h]) for h in range(H)]
    for h in range(H):
        check(dq[0, h].cpu(), refs[h][0], f"bitmap h{h} dq")
    for kh in range(Hkv):
        dk_ref = sum(refs[h][1] for h in range(kh * G, kh * G + G))
        dv_ref = sum(refs[h][2] for h in range(kh * G, kh * G + G))
        check(dk[0, kh].cpu(), dk_ref, f"bitmap kv{kh} dk")
        check(dv[0, kh].cpu(), dv_ref, f"bitmap kv{kh} dv")
