"""BlockMask builder on the GPU: integer tables bit-exact against the oracle's
brute-force classification, for every workload mask and for ragged / unsorted cases."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import blockmask as OB

pytestmark = pytest.mark.gpu


def _gpu_tables(kind, L, S, window=0, doc=None):
    import block_sparse_attention_create_b200 as fa
    dd = doc.to("cuda") if doc is not None else None
    bm = fa.create_block_mask(kind, L, S, window=window, doc_id=dd, device="cuda")
    torch.cuda.synchronize()
    return bm.tables()


def _check(kind, L, S, window=0, doc=None):
    got = _gpu_tables(kind, L, S, window, doc)
    ref = OB.block_tables(kind, L, S, window or None, None if doc is None else doc.numpy())
    for key in ("kv_num_blocks", "kv_indices", "full_kv_num_blocks", "full_kv_indices"):
        assert np.array_equal(got[key].reshape(ref[key].shape), ref[key]), key
    # schedule: a permutation of the rows, by descending live count, ties ascending,
    # each with its partial / full counts
    cnt = ref["kv_num_blocks"] + ref["full_kv_num_blocks"]
    order = got["q_order"][0::2]
    packed = got["q_order"][1::2]
    assert sorted(order.tolist()) == list(range(len(cnt)))
    keys = [(-int(cnt[i]), int(i)) for i in order]
    assert keys == sorted(keys)
    assert np.array_equal(packed & 0xFFFF, ref["kv_num_blocks"][order])
    assert np.array_equal(packed >> 16, ref["full_kv_num_blocks"][order])


@pytest.mark.parametrize("w", W.ALL, ids=lambda w: w.name)
def test_workload_tables_bit_exact(w):
    _check(w.mask_kind, w.L, w.S, w.window, W.make_doc_id(w))


@pytest.mark.parametrize("kind,L,S,window", [
    (0, 1, 1, 0), (0, 129, 129, 0), (0, 300, 1000, 0), (0, 1000, 300, 0), (0, 5, 0, 0),
    (1, 1000, 1000, 1), (1, 1000, 1000, 127), (1, 1000, 1000, 129), (1, 700, 300, 50),
    (1, 4096, 4096, 10 ** 9), (2, 1000, 1000, 0), (2, 384, 200, 0)])
def test_ragged_tables_bit_exact(kind, L, S, window):
    doc = None
    if kind == 2:
        g = torch.Generator().manual_seed(L + S)
        doc = torch.randint(0, 4, (max(L, S),), generator=g, dtype=torch.int32)  # unsorted
    _check(kind, L, S, window, doc)


@pytest.mark.parametrize("pattern", ["random300", "descending_runs", "stride37", "one_per_block_end"])
def test_document_tables_many_ids(pattern):
    """Document classification with many distinct ids per block (each distinct key id
    of a block takes one pass in the builder) and with ids whose only matches lie
    above the causal diagonal (q < k), against the brute-force oracle."""
    L = S = 1000
    pos = torch.arange(L, dtype=torch.int32)
    if pattern == "random300":
        doc = torch.randint(0, 300, (L,), generator=torch.Generator().manual_seed(7), dtype=torch.int32)
    elif pattern == "descending_runs":
        doc = (L - 1 - pos) // 50
    elif pattern == "stride37":
        doc = pos % 37
    else:  # each block's last key shares its id with only the next block's first query
        doc = pos.clone()
        doc[127::128] = -1 - (pos[127::128] // 128)
        doc[128::128] = -1 - (pos[128::128] // 128 - 1)
    _check(2, L, S, 0, doc.to(torch.int32))


def test_page1_densities_from_gpu_tables(golden):
    """The densities printed on page 1, recomputed from the GPU's tables."""
    for pattern, seq, window, _, blk_pct in golden("page1_density_table.txt"):
        L = int(seq)
        kind, wdw = (0, 0) if pattern == "causal" else (1, int(window))
        t = _gpu_tables(kind, L, L, wdw)
        live = int(t["kv_num_blocks"].sum() + t["full_kv_num_blocks"].sum())
        nq = len(t["kv_num_blocks"])
        assert f"{100 * live / (nq * nq):.2f}" == blk_pct
