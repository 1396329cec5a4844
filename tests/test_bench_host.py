"""Host-side figures of bench.py (no GPU): the live-block counts it credits FLOPs
for come from closed forms and a pass over the document ids / bitmap words; they
must equal the oracle's pair-by-pair block classification exactly, and the
decode pair counts must equal the oracle's lower-right masks."""
import numpy as np
import pytest

import bench
import workloads as W
from oracle import blockmask as OB
from oracle import masks as OM

_KIND = {W.MASK_CAUSAL: OM.CAUSAL, W.MASK_SLIDING_WINDOW_CAUSAL: OM.SLIDING_WINDOW_CAUSAL,
         W.MASK_DOCUMENT_CAUSAL: OM.DOCUMENT_CAUSAL, W.MASK_BITMAP: OM.BITMAP}


@pytest.mark.parametrize("name", [n for n, w in W.BY_NAME.items()
                                  if not bench.is_decode(w) and w.L <= 16384])
def test_live_blocks_match_oracle_classification(name):
    w = W.BY_NAME[name]
    doc = W.make_doc_id(w)
    live, _, _ = OB.classify(_KIND[w.mask_kind], w.L, w.S, window=w.window or None,
                             doc_id=None if doc is None else doc.numpy(),
                             bitmap=W.make_bitmap(w))
    np.testing.assert_array_equal(bench.live_blocks_per_row(w), live.sum(axis=1))


def test_benchmark_workload_figures():
    """Window 256 at 32768, B1 H8 D64: 765 live blocks (page-1 density 1.17%),
    4 * 64 * 128^2 * 765 * 8 FLOPs, and Q, K, V, out once plus LSE and tables."""
    w = W.BY_NAME["swa256_L32768_B1_H8_D64_bf16"]
    fig = bench.work_figures(w)
    assert fig["live_blocks"] == 765
    assert fig["flops"] == 4 * 64 * 128 * 128 * 765 * 8
    tensors = 8 * 32768 * 64 * 2 * 4 + 8 * 32768 * 4
    assert tensors <= fig["bytes"] <= tensors + 256 * (3 + 2 * 256) * 4


def test_grouped_query_bytes_count_each_kv_head_once():
    w = W.BY_NAME["gqa_causal_L8192_B1_H32_Hkv8_D64_bf16"]
    fig = bench.work_figures(w)
    qo = 32 * 8192 * 64 * 2 * 2 + 32 * 8192 * 4
    kv = 8 * 8192 * 64 * 2 * 2
    assert qo + kv <= fig["bytes"] <= qo + kv + 64 * (3 + 2 * 64) * 4


@pytest.mark.parametrize("kind,L,S,window", [(W.MASK_DECODE_FULL, 3, 100, 0),
                                             (W.MASK_DECODE_CAUSAL, 5, 300, 0),
                                             (W.MASK_DECODE_CAUSAL, 1, 32768, 0),
                                             (W.MASK_DECODE_SLIDING_WINDOW, 7, 200, 50),
                                             (W.MASK_DECODE_SLIDING_WINDOW, 4, 3, 2)])
def test_decode_pairs_match_lower_right_masks(kind, L, S, window):
    import torch
    w = W.Workload(name="adhoc_decode", B=1, H=1, L=L, S=S, D=64, dtype=torch.bfloat16,
                   mask_kind=kind, window=window)
    m = OM.mask_rows(kind, np.arange(L), S, window or None, q_len=L)
    np.testing.assert_array_equal(bench.decode_pairs_per_row(w), m.sum(axis=1))


def test_replica_launcher_and_max_over_ranks_on_cpu():
    """`bench.py --gpus 2` without an outer launcher starts two ranks itself
    (torch.distributed.run, 127.0.0.1), they rendezvous over gloo, and the job's
    time is the slowest rank's: rank 1 steps twice as long as rank 0, so the
    reported time per step is rank 1's and n_gpus is the number of ranks."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                        "--dry-run", "--steps", "5"], capture_output=True, text=True, env=env,
                       timeout=240)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout   # rank 0 alone prints
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and len(d["rank_ms"]) == 2
    assert d["rank_ms"][1] > d["rank_ms"][0]
    assert abs(d["ms_per_step"] * d["steps"] - max(d["rank_ms"])) < 1e-6
    assert abs(d["value"] - 2 * 5 / (max(d["rank_ms"]) * 1e-3)) < 1e-6


def test_ranks_must_match_gpus():
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                        "--dry-run"], capture_output=True, text=True, env=env, timeout=120)
    assert r.returncode != 0 and "ranks were launched" in r.stderr
