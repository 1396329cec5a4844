"""fa_flex_attention_fwd_noalloc: the allocation-free mask build + forward, whose
block tables and error word live in the library's static device scratch.

Its output must equal, bit for bit, the output of the existing entry points
(fa_create_block_mask + fa_flex_attention_fwd with caller-owned tables and
workspace) on the same inputs -- both run the same kernels on the same tables.
Collected last so that it also runs after every other test in one process."""
import ctypes
import os
import subprocess
import tempfile

import pytest
import torch

import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fa():
    from block_sparse_attention_create_b200 import _binding
    return _binding


def test_scratch_limit_matches_header():
    fa = _fa()
    src = ('#include <stdio.h>\n#include "fa.h"\n'
           'int main(void){printf("%zu\\n", FA_NOALLOC_SCRATCH_BYTES); return 0;}\n')
    with tempfile.TemporaryDirectory() as d:
        c, exe = os.path.join(d, "p.c"), os.path.join(d, "p")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        val = int(subprocess.run([exe], capture_output=True, text=True, check=True).stdout)
    assert val == fa.FA_NOALLOC_SCRATCH_BYTES == 4 << 20


def test_rejects_problems_beyond_the_scratch_before_any_cuda_call():
    """723 x 723 blocks fill the 4 MiB exactly; 724 x 724 do not.  The size check
    precedes every CUDA call, so this runs without a GPU."""
    fa = _fa()
    null = ctypes.c_void_p(0)
    def call(L, S):
        return fa.fa_flex_attention_fwd_noalloc(null, null, null, fa.FA_BF16, 1, 1, L, S, 64,
                                                fa.FA_MASK_CAUSAL, 0, null, fa.FA_SCORE_NONE,
                                                0.0, 0.0, null, null, null, null)
    assert call(724 * 128, 724 * 128) == fa.FA_ERR_SCRATCH_TOO_SMALL
    assert call(1024 * 128, 600 * 128) == fa.FA_ERR_SCRATCH_TOO_SMALL
    assert call(1024 * 128, 16) == fa.FA_ERR_INVALID_ARG  # 1024 x 1 blocks fit
    # fits: rejected only later, for the NULL tensors
    assert call(723 * 128, 723 * 128) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_status_string(fa.FA_ERR_SCRATCH_TOO_SMALL) == b"FA_ERR_SCRATCH_TOO_SMALL"


def _existing_path(fa, q, k, v, kind, window, doc, sk, cap):
    bm = fa.create_block_mask(kind, q.shape[2], k.shape[2], window=window, doc_id=doc,
                              device="cuda")
    return fa.flex_attention(q, k, v, bm, score_mod=sk, softcap=cap, return_lse=True)


@pytest.mark.gpu
def test_noalloc_equals_existing_entry_points_on_two_calls_in_a_row():
    fa = _fa()
    g = torch.Generator().manual_seed(23)
    doc = torch.randint(0, 5, (2000,), generator=g, dtype=torch.int32).sort().values.cuda()
    cases = [  # (q, k, v, mask kind, window, doc_id, score_mod, softcap)
        (*(t.cuda() for t in W.random_qkv(2, 4, 1000, 1000, 64, torch.bfloat16, seed=21)),
         fa.FA_MASK_SLIDING_WINDOW_CAUSAL, 300, None, fa.FA_SCORE_NONE, 0.0),
        (*(t.cuda() for t in W.random_qkv(1, 3, 2000, 2000, 128, torch.float16, seed=22)),
         fa.FA_MASK_DOCUMENT_CAUSAL, 0, doc, fa.FA_SCORE_TANH_SOFTCAP, 30.0),
    ]
    refs = [_existing_path(fa, *c) for c in cases]
    torch.cuda.synchronize()
    assert fa.last_device_error() == fa.FA_OK

    err = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    got = []
    for i, (q, k, v, kind, window, d, sk, cap) in enumerate(cases):
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
        # back to back on one stream: the second call reuses the scratch the first used
        got.append(fa.flex_attention_noalloc(q, k, v, kind, window=window, doc_id=d,
                                             score_mod=sk, softcap=cap, lse=lse,
                                             device_error=err[i:i + 1]))
    torch.cuda.synchronize()
    assert err.tolist() == [0, 0]
    for (o, l), (ro, rl) in zip(got, refs):
        assert torch.equal(o, ro)
        assert torch.equal(l, rl)


@pytest.mark.gpu
def test_noalloc_causal_at_the_scratch_limit():
    """Causal masks, and a problem whose tables fill the scratch to its last block
    (L = S = 723 * 128: 723 x 723 blocks), equal the existing entry points bit for
    bit, twice in a row."""
    fa = _fa()
    L = 723 * 128
    cases = [(*(t.cuda() for t in W.random_qkv(1, 3, 1500, 1500, 64, torch.bfloat16, seed=24)),),
             (*(t.cuda() for t in W.random_qkv(1, 1, L, L, 64, torch.bfloat16, seed=25)),)]
    err = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    for n, (q, k, v) in enumerate(cases):
        ro, rl = _existing_path(fa, q, k, v, fa.FA_MASK_CAUSAL, 0, None, fa.FA_SCORE_NONE, 0.0)
        for rep in range(2):
            o, l = fa.flex_attention_noalloc(q, k, v, fa.FA_MASK_CAUSAL,
                                             device_error=err[2 * n + rep:2 * n + rep + 1])
            torch.cuda.synchronize()
            assert torch.equal(o, ro) and torch.equal(l, rl), (n, rep)
    assert err.tolist() == [0, 0, 0, 0]
