"""fa_block_mask_validate: the host-side check of block tables the forward kernel
would otherwise trust.  Correct tables (from the CPU oracle's classification, with
the schedule written out from its definition: rows by descending live count, ties
by ascending row) pass; each planted corruption is caught and the offending row
reported.  No GPU: the check reads host arrays only."""
import numpy as np
import pytest

import workloads as W
from oracle import blockmask as OB


@pytest.fixture(scope="module")
def fa():
    from block_sparse_attention_create_b200 import _binding
    return _binding


def _tables(kind, L, S, window=None, doc=None):
    keys = ("kv_num_blocks", "kv_indices", "full_kv_num_blocks", "full_kv_indices")
    bt = OB.block_tables(kind, L, S, window=window, doc_id=doc)
    t = {k: np.array(bt[k], dtype=np.int32) for k in keys}
    n = t["kv_num_blocks"] + t["full_kv_num_blocks"]
    rows = sorted(range(len(n)), key=lambda r: (-int(n[r]), r))
    order = np.zeros(2 * len(n), dtype=np.int32)
    for k, r in enumerate(rows):
        order[2 * k] = r
        order[2 * k + 1] = int(t["kv_num_blocks"][r]) | (int(t["full_kv_num_blocks"][r]) << 16)
    t["q_order"] = order
    return t


CASES = [(W.MASK_CAUSAL, 700, 700, None, None),
         (W.MASK_SLIDING_WINDOW_CAUSAL, 1000, 900, 300, None),
         (W.MASK_DOCUMENT_CAUSAL, 640, 640, None, np.repeat(np.arange(5), 128).astype(np.int32))]


@pytest.mark.parametrize("case", CASES, ids=["causal", "window", "documents"])
def test_correct_tables_pass(fa, case):
    kind, L, S, window, doc = case
    t = _tables(kind, L, S, window, doc)
    nq, nkv = -(-L // 128), -(-S // 128)
    assert fa.validate_tables(t, nq, nkv) == (fa.FA_OK, -1)


def _corrupt(t, what):
    t = {k: v.copy() for k, v in t.items()}
    row = 3
    npart = int(t["kv_num_blocks"][row])
    nfull = int(t["full_kv_num_blocks"][row])
    assert npart >= 1 and nfull >= 2
    if what == "count_above_nkv":
        t["kv_num_blocks"][row] = t["kv_indices"].shape[1] + 1
    elif what == "negative_count":
        t["full_kv_num_blocks"][row] = -1
    elif what == "index_out_of_range":
        t["full_kv_indices"][row, 0] = t["kv_indices"].shape[1]
    elif what == "negative_index":
        t["kv_indices"][row, 0] = -5
    elif what == "not_ascending":
        a = t["full_kv_indices"][row]
        a[0], a[1] = a[1], a[0]
    elif what == "in_both_lists":
        t["full_kv_indices"][row, 0] = t["kv_indices"][row, 0]
    elif what == "nonzero_padding":
        t["kv_indices"][row, npart] = 1
    elif what == "count_without_entries":   # the counts and the lists disagree
        t["kv_num_blocks"][row] = npart + 1
    return t, row


@pytest.mark.parametrize("what", ["count_above_nkv", "negative_count", "index_out_of_range",
                                  "negative_index", "not_ascending", "in_both_lists",
                                  "nonzero_padding", "count_without_entries"])
def test_row_corruptions_are_caught(fa, what):
    t = _tables(W.MASK_CAUSAL, 1024, 1024)
    bad, row = _corrupt(t, what)
    assert fa.validate_tables(bad, 8, 8) == (fa.FA_ERR_INVALID_ARG, row)


def test_schedule_corruptions_are_caught(fa):
    t = _tables(W.MASK_CAUSAL, 1024, 1024)
    assert fa.validate_tables(t, 8, 8)[0] == fa.FA_OK
    # a row listed twice (row 7 in place of row 6)
    bad = {k: v.copy() for k, v in t.items()}
    bad["q_order"][2] = bad["q_order"][0]
    bad["q_order"][3] = bad["q_order"][1]
    assert fa.validate_tables(bad, 8, 8)[0] == fa.FA_ERR_INVALID_ARG
    # a row out of range
    bad = {k: v.copy() for k, v in t.items()}
    bad["q_order"][4] = 8
    assert fa.validate_tables(bad, 8, 8)[0] == fa.FA_ERR_INVALID_ARG
    # counts that disagree with the row's lists (more partial blocks than listed)
    bad = {k: v.copy() for k, v in t.items()}
    bad["q_order"][1] += 1
    assert fa.validate_tables(bad, 8, 8)[0] == fa.FA_ERR_INVALID_ARG
    # out of order: two ranks swapped
    bad = {k: v.copy() for k, v in t.items()}
    o = bad["q_order"].reshape(-1, 2)
    o[[0, 1]] = o[[1, 0]]
    assert fa.validate_tables(bad, 8, 8)[0] == fa.FA_ERR_INVALID_ARG


def test_instances_and_argument_errors(fa):
    """Per-(batch, head) tables, instance-major: a corruption in instance 2 is
    reported as 2 * nQ + row; bad sizes and missing arrays are argument errors."""
    parts = [_tables(W.MASK_SLIDING_WINDOW_CAUSAL, 1024, 1024, 128 * (i + 1)) for i in range(3)]
    t = {k: np.concatenate([p[k] for p in parts]) for k in parts[0]}
    assert fa.validate_tables(t, 8, 8, instances=3) == (fa.FA_OK, -1)
    bad = {k: v.copy() for k, v in t.items()}
    bad["kv_indices"][2 * 8 + 5, 0] = 99
    assert fa.validate_tables(bad, 8, 8, instances=3) == (fa.FA_ERR_INVALID_ARG, 2 * 8 + 5)
    assert fa.validate_tables(t, 8, 8, instances=0)[0] == fa.FA_ERR_INVALID_ARG
    assert fa.validate_tables(t, -1, 8)[0] == fa.FA_ERR_INVALID_ARG
    import ctypes
    null = ctypes.c_void_p(0)
    assert fa.fa_block_mask_validate(null, null, null, null, null, 8, 8, 1, None) == \
        fa.FA_ERR_INVALID_ARG
    assert fa.fa_block_mask_validate(null, null, null, null, null, 0, 8, 1, None) == fa.FA_OK
