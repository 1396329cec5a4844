"""Backward pass on the GPU (dQ, dK, dV recomputed over the BlockMask from the
forward's LSE) against the fp64 CPU oracle's gradients: element by element on
small ragged shapes, and on sampled rows of the full-size benchmark workloads.

Tolerance (derived).  Three sources of error:
  - fp32 accumulation and the 16-bit store of dq / dk / dv (unit roundoff u =
    2^-8 for bf16, 2^-11 for fp16): covered by 2e-2 * (|ref| + rms(ref)), rms
    over the tensor;
  - P and dS enter the tensor-core products in the input dtype, each element
    rounded (|error| <= u |x|, independent): their sums carry at most
    3 * u * sqrt(sum of squared terms) (three times the root-sum-square, ~5
    standard deviations of the uniform rounding error), e.g. for dv_j
    3u * sqrt(sum_i P_ij^2 dO_i^2) and for dk_j 3u * scale * sqrt(sum_i dS_ij^2 q_i^2);
  - the row sums delta_i = rowsum(dO_i * O_i) use the STORED 16-bit forward output.
    Each O_id carries the forward's 16-bit P (<= u * (P|V|)_id) and its own
    rounding (<= u |O_id|), so |dO_id| * 2u * (P|V|)_id bounds each term's error;
    the D terms round independently, so their root-sum-square
    A_i = 2u * ||dO_i * (P|V|)_i||_2 stands for |d delta_i|.  It enters
    dS_ij = P_ij (dO_i . v_j - delta_i) (* 1 - tanh^2 <= 1) as P_ij * A_i, hence
        |d dq_i| <= scale * A_i * (P |K|)_i,   |d dk_j| <= scale * (P^T (A * |Q|))_j
    (dk summed over the query heads of a group; dv does not use delta).  On
    near one-hot rows dO_i . v_j - delta_i cancels, and this term dominates
    there.
Each element must satisfy |err| <= 2e-2 * (|ref| + rms) + its two terms + 1e-6."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import attention as OA
from oracle import backward as OBW
from oracle import masks as OM

pytestmark = pytest.mark.gpu


def _check_grad(got, ref, prop, what):
    got = got.double().numpy()
    rms = float(np.sqrt((ref ** 2).mean())) if ref.size else 0.0
    err = np.abs(got - ref)
    bound = 2e-2 * (np.abs(ref) + rms) + prop + 1e-6
    assert np.isfinite(got).all(), what
    assert (err <= bound).all(), f"{what}: worst {(err / bound).max():.2f} x bound"


def _run(B, H, Hkv, L, S, D, dtype, kind, window=0, doc=None, words=None, sk=0, cap=0.0, seed=0):
    import block_sparse_attention_create_b200 as fa
    q, k, v = W.random_qkv(B, H, L, S, D, dtype, seed=seed, Hkv=Hkv)
    g = torch.Generator().manual_seed(seed + 1)
    dout = torch.randn(B, H, L, D, generator=g).to(dtype)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, dout))
    bits = (torch.from_numpy(np.ascontiguousarray(words).view(np.int32)).cuda()
            if words is not None else None)
    bm = fa.create_block_mask(kind, L, S, window=window,
                              doc_id=doc.cuda() if doc is not None else None, bitmap=bits)
    out, lse = fa.flex_attention(qd, kd, vd, bm, score_mod=sk, softcap=cap, return_lse=True)
    dq, dk, dv = fa.flex_attention_backward(qd, kd, vd, out, dod, lse, bm, score_mod=sk,
                                            softcap=cap, check=True)
    torch.cuda.synchronize()
    assert fa.last_device_error() == fa.FA_OK
    dq, dk, dv = dq.cpu(), dk.cpu(), dv.cpu()
    G = H // Hkv
    u = 2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -11
    scale = 1.0 / np.sqrt(D)
    for b in range(B):
        dk_ref = np.zeros((Hkv, S, D))
        dv_ref = np.zeros((Hkv, S, D))
        dk_prop = np.zeros((Hkv, S, D))
        dk_rss = np.zeros((Hkv, S, D))
        dv_rss = np.zeros((Hkv, S, D))
        for h in range(H):
            kh = OA.kv_head(h, H, Hkv)
            rq, rk, rv, p, ds = OBW.attention_head_backward(
                q[b, h], k[b, kh], v[b, kh], dout[b, h], kind, window=window or None,
                doc_id=None if doc is None else doc.numpy(), score_kind=sk, softcap=cap,
                bitmap=words, return_probs=True)
            qa, ka, va, ga = (np.abs(t.double().numpy()) for t in (q[b, h], k[b, kh], v[b, kh],
                                                                   dout[b, h]))
            A = 2 * u * np.sqrt(((ga * (p @ va)) ** 2).sum(axis=1))
            ds2 = ds ** 2
            _check_grad(dq[b, h], rq, scale * A[:, None] * (p @ ka)
                        + 3 * u * scale * np.sqrt(ds2 @ ka ** 2), f"dq b{b} h{h}")
            dk_ref[kh] += rk
            dv_ref[kh] += rv
            dk_prop[kh] += scale * (p.T @ (A[:, None] * qa))
            dk_rss[kh] += scale ** 2 * (ds2.T @ qa ** 2)
            dv_rss[kh] += (p ** 2).T @ ga ** 2
        for kh in range(Hkv):
            _check_grad(dk[b, kh], dk_ref[kh], dk_prop[kh] + 3 * u * np.sqrt(dk_rss[kh]),
                        f"dk b{b} g{kh} (group of {G})")
            _check_grad(dv[b, kh], dv_ref[kh], 3 * u * np.sqrt(dv_rss[kh]), f"dv b{b} g{kh}")


@pytest.mark.parametrize("L,S,D,dtype,kind,window", [
    (300, 300, 64, torch.bfloat16, OM.CAUSAL, 0), (333, 200, 128, torch.float16, OM.SLIDING_WINDOW_CAUSAL, 100),
    (200, 333, 64, torch.bfloat16, OM.CAUSAL, 0), (257, 257, 128, torch.bfloat16, OM.CAUSAL, 0)])
def test_backward_rules(L, S, D, dtype, kind, window):
    _run(2, 2, 2, L, S, D, dtype, kind, window, seed=L + S)


def test_backward_documents_and_bitmap():
    doc = torch.randint(0, 3, (400,), generator=torch.Generator().manual_seed(4), dtype=torch.int32)
    _run(1, 2, 2, 400, 400, 64, torch.bfloat16, OM.DOCUMENT_CAUSAL, doc=doc, seed=5)
    words = W.random_bitmap(300, 260, seed=6)
    _run(1, 2, 2, 300, 260, 64, torch.bfloat16, OM.BITMAP, words=words, seed=7)


def test_backward_softcap_and_grouped_heads():
    _run(1, 4, 2, 256, 256, 128, torch.bfloat16, OM.CAUSAL, sk=1, cap=5.0, seed=8)
    _run(1, 4, 1, 300, 300, 64, torch.float16, OM.SLIDING_WINDOW_CAUSAL, window=64, seed=9)


@pytest.mark.parametrize("name,heads,q_rows,k_rows", [
    ("swa256_L32768_B1_H8_D64_bf16", (5,), [*range(0, 64), *range(20000, 20064)],
     [*range(1000, 1064), *range(32704, 32768)]),
    ("causal_L8192_B1_H8_D64_bf16", (0, 7), [*range(0, 64), *range(8128, 8192)],
     [*range(8064, 8192)])])
def test_backward_full_size_sampled(name, heads, q_rows, k_rows):
    """The backward workloads bench.py --backward times, at full size and with its
    inputs: all heads computed on the GPU in one call; sampled rows of dq and of
    dk / dv against the oracle's sampled gradients, with the tolerance derived above
    (its terms from the sampled rows of P and dS)."""
    import block_sparse_attention_create_b200 as fa
    w = W.BY_NAME[name]
    q, k, v = W.make_qkv(w)
    g = torch.Generator().manual_seed(w.seed + 1)
    dout = torch.randn(q.shape, generator=g).to(q.dtype)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, dout))
    bm = fa.create_block_mask(w.mask_kind, w.L, w.S, window=w.window)
    out, lse = fa.flex_attention(qd, kd, vd, bm, return_lse=True)
    dq, dk, dv = fa.flex_attention_backward(qd, kd, vd, out, dod, lse, bm)
    torch.cuda.synchronize()
    assert fa.last_device_error() == fa.FA_OK
    kind = {W.MASK_CAUSAL: OM.CAUSAL, W.MASK_SLIDING_WINDOW_CAUSAL: OM.SLIDING_WINDOW_CAUSAL}[
        w.mask_kind]
    u = 2.0 ** -8 if q.dtype == torch.bfloat16 else 2.0 ** -11
    scale = 1.0 / np.sqrt(w.D)
    for h in heads:
        res = OBW.attention_head_backward_sampled(q[0, h], k[0, h], v[0, h], dout[0, h], kind,
                                                  q_rows, k_rows, window=w.window or None)
        rows, p, ds = res["rows"], res["p"], res["ds"]
        ka, va = (np.abs(t[0, h].double().numpy()) for t in (k, v))
        qa, ga = (np.abs(t[0, h].double().numpy()[rows]) for t in (q, dout))
        A = 2 * u * np.sqrt(((ga * (p @ va)) ** 2).sum(axis=1))
        at = np.searchsorted(rows, q_rows)
        dq_prop = (scale * A[at, None] * (p[at] @ ka)
                   + 3 * u * scale * np.sqrt(ds[at] ** 2 @ ka ** 2))
        pk, dsk = p[:, k_rows], ds[:, k_rows]
        dk_prop = scale * (pk.T @ (A[:, None] * qa)) + 3 * u * scale * np.sqrt(dsk.T ** 2 @ qa ** 2)
        dv_prop = 3 * u * np.sqrt(pk.T ** 2 @ ga ** 2)
        _check_grad(dq[0, h].cpu()[q_rows], res["dq"], dq_prop, f"{name} dq h{h}")
        _check_grad(dk[0, h].cpu()[k_rows], res["dk"], dk_prop, f"{name} dk h{h}")
        _check_grad(dv[0, h].cpu()[k_rows], res["dv"], dv_prop, f"{name} dv h{h}")
