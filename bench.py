"""Benchmark of the block-sparse attention hot path on B200.

A step is one pass of the whole path over one batch of synthetic input:
fa_create_block_mask (block classification + schedule order) followed by
fa_flex_attention_fwd.  Default workload: sliding-window causal W=256,
B=1 H=8 L=S=32768 D=64 bf16 (the FlexAttention vs SDPA M1 Max benchmark's
longest case, qiita kiarina, "検証結果").

Prints one JSON line (rank 0).  `value` is live-block TFLOP/s of whole steps
(4 * D * 128^2 FLOPs per live block per batch*head: the two matmuls over the
blocks the mask keeps; skipped blocks count nothing), summed over ranks and
divided by the max-over-ranks device time.  L2 is flushed (a 512 MiB write)
between timed steps, outside the timed region.

--impl reference times the CPU fp64 oracle (the only reference there is) on a
bounded row sample of the same workload, on this host's cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "fwd ms & live-block TFLOP/s (frac of BF16 TC peak) at S=32768 W=256"
UNIT = "TFLOP/s"
# Page-1 FlexAttention forward on M1 Max at this workload: 75.27 ms (context only).
PAGE_FWD_MS = {"swa256_L32768_B1_H8_D64_bf16": 75.27, "causal_L8192_B1_H8_D64_bf16": 231.22,
               "swa64_L8192_B1_H8_D64_bf16": 11.75, "swa256_L8192_B1_H8_D64_bf16": 19.14,
               "swa1024_L8192_B1_H8_D64_bf16": 56.24, "swa4096_L8192_B1_H8_D64_bf16": 169.24}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (read + write) of one launch of the dominant kernel from an ncu capture,
# per workload, with the hash of the kernel's device code it was taken on (each .cu
# file up to its "host side" marker, and the PTX helpers): reported as
# roofline.traffic only while the device code still hashes to that value (null once
# the kernel changed).
FWD_SOURCES = ("block_sparse_attention_create_b200/csrc/fwd_sm100.cu",
               "block_sparse_attention_create_b200/csrc/sm100_ptx.cuh")
DECODE_SOURCES = ("block_sparse_attention_create_b200/csrc/decode.cu",
                  "block_sparse_attention_create_b200/csrc/sm100_ptx.cuh")
NCU_TRAFFIC = {
    "swa256_L32768_B1_H8_D64_bf16": {
        "bytes": 101080576 + 7429376, "sources": FWD_SOURCES,
        "sources_sha256": "0e33e5c29e978af55a7630c50c2c7c1d314fa86b85e0778dde788592b50e0683",
        "summary": "profiles/fwd_kernel_swa256_L32768_B1_H8_D64_launches.md"},
    "decode_L1_S32768_B8_H32_Hkv8_D128_bf16": {
        "bytes": 1073856512 + 3907840, "sources": DECODE_SOURCES,
        "sources_sha256": "7a50235ad66ea70215c719a32ac78bf42221f867fdc26866fef91ca8c4df4d1a",
        "summary": "profiles/decode_mma_kernel_L1_S32768_B8_H32_Hkv8_D128_full.md"},
}


HOST_MARKER = b"// ---------------------------------------------------------------- host side"


def kernel_sources_hash(sources):
    """sha256 of the device code: each .cu source up to its host-side marker (the
    whole file if it has none), and every header whole."""
    import hashlib
    h = hashlib.sha256()
    for rel in sources:
        with open(os.path.join(ROOT, rel), "rb") as f:
            data = f.read()
        if rel.endswith(".cu") and HOST_MARKER in data:
            data = data[:data.index(HOST_MARKER)]
        h.update(data)
    return h.hexdigest()


def ncu_traffic(w: W.Workload):
    rec = NCU_TRAFFIC.get(w.name)
    if rec is None or rec["sources_sha256"] != kernel_sources_hash(rec["sources"]):
        return None
    return rec["bytes"]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def live_blocks_per_row(w: W.Workload):
    """Live 128x128 blocks of every q-block row, from the GPU-independent closed
    forms of the mask (causal / window) or a pass over the document ids."""
    nq = -(-w.L // 128)
    nkv = -(-w.S // 128)
    out = np.zeros(nq, dtype=np.int64)
    doc = W.make_doc_id(w)
    doc = doc.numpy() if doc is not None else None
    words = W.make_bitmap(w)
    if words is not None:  # a block is live if any of its words has a bit set
        tail = np.uint32((1 << (w.S % 32)) - 1) if w.S % 32 else np.uint32(0xFFFFFFFF)
        words = words.copy()
        if w.S % 32:
            words[:, w.S // 32] &= tail
        words[:, -(-w.S // 32):] = 0
        blk = np.zeros((nq * 128, nkv * 4), dtype=np.uint32)
        blk[: w.L] = words
        any_bit = blk.reshape(nq, 128, nkv, 4).any(axis=(1, 3))
        return any_bit.sum(axis=1).astype(np.int64)
    for i in range(nq):
        q0, q1 = i * 128, min(w.L, i * 128 + 128) - 1
        for j in range(nkv):
            k0, k1 = j * 128, min(w.S, j * 128 + 128) - 1
            if k0 > q1:
                break
            if w.mask_kind == W.MASK_SLIDING_WINDOW_CAUSAL and k1 < q0 - w.window + 1:
                continue
            if w.mask_kind == W.MASK_DOCUMENT_CAUSAL:
                dq = set(doc[q0:q1 + 1].tolist())
                if not dq.intersection(doc[k0:k1 + 1].tolist()):
                    continue
            out[i] += 1
    return out


def decode_pairs_per_row(w: W.Workload):
    """Keys each of the L new queries sees (decode, lower-right alignment)."""
    pos = w.S - w.L + np.arange(w.L)          # key position of each query
    if w.mask_kind == W.MASK_DECODE_FULL:
        return np.full(w.L, w.S, dtype=np.int64)
    hi = np.clip(pos + 1, 0, w.S)              # keys 0 .. pos
    if w.mask_kind == W.MASK_DECODE_CAUSAL:
        return hi.astype(np.int64)
    return np.clip(hi - np.clip(pos - w.window + 1, 0, None), 0, None).astype(np.int64)


def is_decode(w: W.Workload) -> bool:
    return w.mask_kind >= W.MASK_DECODE_FULL


def work_figures(w: W.Workload):
    if is_decode(w):
        pairs = decode_pairs_per_row(w)
        flops = 4.0 * w.D * float(pairs.sum()) * w.B * w.H
        bytes_ = (w.B * w.H * w.L * w.D * 2 * 2 + w.B * w.n_kv_heads * w.S * w.D * 2 * 2
                  + w.B * w.H * w.L * 4)
        return {"live_blocks": None, "pairs": pairs, "flops": flops, "bytes": bytes_}
    per_row = live_blocks_per_row(w)
    live = int(per_row.sum())
    flops = 4.0 * w.D * 128 * 128 * live * w.B * w.H
    esz = 2
    bytes_ = (w.B * w.H * (w.L * w.D * esz * 2 + w.L * 4)           # Q, out, LSE
              + w.B * w.n_kv_heads * w.S * w.D * esz * 2              # K, V once per K/V head
              + per_row.size * (3 + 2 * (-(-w.S // 128))) * 4)
    return {"live_blocks": live, "per_row": per_row, "flops": flops, "bytes": bytes_}


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the GPU is busy."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "utilization.gpu")

    def __init__(self, index, enabled=True):
        self.index = index
        self.enabled = enabled
        self.proc = None

    def __enter__(self):
        if not self.enabled:
            return self
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons, busy = [], None, set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                util = float(f[9])
                clk = float(f[1])
                mx = float(f[2])
            except ValueError:
                continue
            if util < 50:
                continue
            busy += 1
            sm.append(clk)
            for n, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples_under_load": busy}


def step_calls(fa, w, qd, kd, vd, dd, bd, out, lse, device, stream):
    """(mask build, forward, device-error query) of one step through the public API.
    Decode workloads have no mask tables: the build is empty."""
    if is_decode(w):
        nbytes = int(fa.fa_decode_workspace_bytes(w.B, w.H, w.n_kv_heads, w.L, w.S, w.D))
        dws = fa.decode_workspace(device, nbytes)

        def attend():
            fa.flex_attention_decode(qd, kd, vd, mask=w.mask_kind - W.MASK_DECODE_FULL,
                                     window=w.window, score_mod=w.score_kind, softcap=w.softcap,
                                     out=out, lse=lse, ws=dws, stream=stream)
        return (lambda: None), attend, (lambda: fa.last_decode_error(device))
    bm = fa.BlockMask(w.L, w.S, device)
    ws = fa.workspace(device)

    def build():
        fa.create_block_mask(w.mask_kind, w.L, w.S, window=w.window, doc_id=dd, out=bm,
                             stream=stream, bitmap=bd)

    def attend():
        fa.flex_attention(qd, kd, vd, bm, score_mod=w.score_kind, softcap=w.softcap, out=out,
                          lse=lse, ws=ws, stream=stream)
    return build, attend, (lambda: fa.last_device_error(device))


def run_ours(args, w: W.Workload, rank, world, device):
    import block_sparse_attention_create_b200 as fa
    torch.cuda.set_device(device)
    q, k, v = W.make_qkv(w)
    doc = W.make_doc_id(w)
    words = W.make_bitmap(w)
    bits = torch.from_numpy(words.view(np.int32)) if words is not None else None
    qd, kd, vd = q.to(device), k.to(device), v.to(device)
    dd = doc.to(device) if doc is not None else None
    bd = bits.to(device) if bits is not None else None
    out = torch.empty_like(qd)
    lse = torch.empty(w.B, w.H, w.L, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=device)
    build, attend, dev_error = step_calls(fa, w, qd, kd, vd, dd, bd, out, lse, device, stream)

    def step():
        build()
        attend()

    fig = work_figures(w)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert dev_error() == fa.FA_OK

    # keep the GPU at load clocks for ~1 s inside the sampling window, untimed
    def events():
        return [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    starts, mids, ends = events(), events(), events()
    t_starts, t_ends = events(), events()
    with ClockSampler(device.index if device.index is not None else 0,
                      enabled=not args.profile) as clk:
        t_end = time.time() + (0.0 if args.profile else 1.0)
        while time.time() < t_end:
            for _ in range(50):
                step()
            torch.cuda.synchronize()
        # Breakdown of a step into mask build and forward (outside the timed region):
        # an event between the two launches also keeps the forward from starting
        # its prologue under the end of the mask build (programmatic dependent
        # launch), so the timed steps below have nothing between them.
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            build()
            mids[i].record(stream)
            attend()
            ends[i].record(stream)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush.zero_()
            t_starts[i].record(stream)
            build()
            attend()
            t_ends[i].record(stream)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
    assert dev_error() == fa.FA_OK
    step_ms = [s.elapsed_time(e) for s, e in zip(t_starts, t_ends)]
    fwd_ms = [m.elapsed_time(e) for m, e in zip(mids, ends)]
    mask_ms = [s.elapsed_time(m) for s, m in zip(starts, mids)]
    total_ms = max_over_ranks(sum(step_ms), device)

    # end to end through the public API: pinned host inputs in, results out
    e2e = ({"ms": float("nan"), "h2d": 0, "d2h": 0} if args.profile
           else run_e2e(args, w, fa, q, k, v, doc, bits, device, world))
    return {"fig": fig, "total_ms": total_ms, "step_ms": step_ms, "fwd_ms": fwd_ms,
            "mask_ms": mask_ms, "clocks": clk.summary(), "e2e": e2e}


def config_sweep(device, steps=10, warmup=3):
    """The forward kernel alone on the other configurations of the benchmark set
    (causal 256, the 8192 sweep, both document workloads, the D = 128 softcap
    workload) and on the workloads of the wider calls (tabulated mask, grouped-query
    heads; decode, whose call is its whole step): mask built once, `warmup`
    launches, then `steps` launches each bracketed by CUDA events with a 512 MiB L2
    flush between them (untimed).  Reported beside the main line so that these
    figures come from the same run."""
    import block_sparse_attention_create_b200 as fa
    peaks, _ = load_peaks()
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    res = {}
    for w in (W.C1_CAUSAL_256, W.C2_CAUSAL_8192) + W.C2_WINDOWS + (
            W.C4_DOC_FIXED, W.C4_DOC_SEEDED, W.C5_SWA1024_SOFTCAP) + W.EXTRA:
        q, k, v = (t.to(device) for t in W.make_qkv(w))
        doc = W.make_doc_id(w)
        dd = doc.to(device) if doc is not None else None
        words = W.make_bitmap(w)
        bd = torch.from_numpy(words.view(np.int32)).to(device) if words is not None else None
        out = torch.empty_like(q)
        lse = torch.empty(w.B, w.H, w.L, dtype=torch.float32, device=device)
        build, attend, dev_error = step_calls(fa, w, q, k, v, dd, bd, out, lse, device, stream)
        build()
        for _ in range(warmup):
            attend()
        torch.cuda.synchronize()
        t = []
        for _ in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            attend()
            e1.record(stream)
            t.append((e0, e1))
        torch.cuda.synchronize()
        assert dev_error() == fa.FA_OK
        ms = sum(a.elapsed_time(b) for a, b in t) / steps
        fig = work_figures(w)
        tflops = fig["flops"] / (ms * 1e-3) / 1e12
        gbs = fig["bytes"] / (ms * 1e-3) / 1e9
        tf, hf = tflops / peaks["bf16_tflops"], gbs / peaks["hbm_gbs"]
        res[w.name] = {"fwd_us": round(ms * 1e3, 2), "live_tflops": round(tflops, 1),
                       "bound": "tensor" if tf >= hf else "hbm", "frac": round(max(tf, hf), 4)}
        del q, k, v, out, lse, bd
    return res


def run_backward(args, w: W.Workload, world, device, fig):
    """Backward step timed like the forward: the mask's column lists and
    fa_flex_attention_bwd, L2 flushed between steps, CUDA events, max over ranks.
    FLOPs credited: 2.5 x the forward's live-block FLOPs (five block products:
    S, dP, dV, dQ, dK against the forward's two)."""
    import block_sparse_attention_create_b200 as fa
    torch.cuda.set_device(device)
    q, k, v = (t.to(device) for t in W.make_qkv(w))
    doc = W.make_doc_id(w)
    dd = doc.to(device) if doc is not None else None
    words = W.make_bitmap(w)
    bd = torch.from_numpy(words.view(np.int32)).to(device) if words is not None else None
    g = torch.Generator().manual_seed(w.seed + 1)
    dout = torch.randn(q.shape, generator=g).to(q.dtype).to(device)
    bm = fa.create_block_mask(w.mask_kind, w.L, w.S, window=w.window, doc_id=dd, device=device,
                              bitmap=bd)
    out, lse = fa.flex_attention(q, k, v, bm, score_mod=w.score_kind, softcap=w.softcap,
                                 return_lse=True)
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=device)

    def step():
        cols = bm.transpose()
        return fa.flex_attention_backward(q, k, v, out, dout, lse, bm, score_mod=w.score_kind,
                                          softcap=w.softcap, columns=cols)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ms = []
    for _ in range(args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        step()
        e1.record()
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    total = max_over_ranks(sum(ms), device)
    flops = 2.5 * fig["flops"]
    peaks, _ = load_peaks()
    tflops = flops * args.steps * world / (total * 1e-3) / 1e12
    line = {"metric": "backward live-block TFLOP/s (2.5 x forward FLOPs)", "value": tflops,
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype_name, "data": "synthetic",
            "config": {**w.describe(), "step": "fa_block_mask_transpose + fa_flex_attention_bwd",
                       "l2": "flushed between timed steps (512 MiB write, untimed)"},
            "roofline": {"bound": "tensor", "achieved": tflops / world, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": tflops / world / peaks["bf16_tflops"],
                         "traffic": None},
            "gpu_launches": 4 * args.steps}
    print(json.dumps(line))


def run_e2e(args, w, fa, q, k, v, doc, bits, device, world):
    hq, hk, hv = (t.pin_memory() for t in (q, k, v))
    hdoc = doc.pin_memory() if doc is not None else None
    hbits = bits.pin_memory() if bits is not None else None
    bd = torch.empty(bits.shape, dtype=bits.dtype, device=device) if bits is not None else None
    hout = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    hlse = torch.empty(w.B, w.H, w.L, dtype=torch.float32).pin_memory()
    qd, kd, vd = (torch.empty(t.shape, dtype=t.dtype, device=device) for t in (q, k, v))
    dd = torch.empty(doc.shape, dtype=doc.dtype, device=device) if doc is not None else None
    out = torch.empty_like(qd)
    lse = torch.empty(w.B, w.H, w.L, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()
    build, attend, _ = step_calls(fa, w, qd, kd, vd, dd, bd, out, lse, device, stream)

    def step():
        qd.copy_(hq, non_blocking=True)
        kd.copy_(hk, non_blocking=True)
        vd.copy_(hv, non_blocking=True)
        if dd is not None:
            dd.copy_(hdoc, non_blocking=True)
        if bd is not None:
            bd.copy_(hbits, non_blocking=True)
        build()
        attend()
        hout.copy_(out, non_blocking=True)
        hlse.copy_(lse, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), device)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv)) + (
        hdoc.numel() * 4 if hdoc is not None else 0) + (hbits.numel() * 4 if hbits is not None else 0)
    d2h = hout.numel() * hout.element_size() + hlse.numel() * 4
    return {"ms": ms, "h2d": h2d, "d2h": d2h}


def oracle_sample(w: W.Workload, rows, fig):
    """Time the oracle on `rows` of head (0, 0); returns (seconds, live FLOPs credited)."""
    from oracle import attention as OA
    q, k, v = W.make_qkv(w)
    doc = W.make_doc_id(w)
    words = W.make_bitmap(w)
    if is_decode(w):  # every new query of the first `rows` heads
        t0 = time.perf_counter()
        for h in range(len(rows)):
            g = OA.kv_head(h, w.H, w.n_kv_heads)
            OA.attention_head(q[0, h], k[0, g], v[0, g], w.mask_kind, window=w.window or None,
                              score_kind=w.score_kind, softcap=w.softcap)
        dt = time.perf_counter() - t0
        return dt, 4.0 * w.D * float(fig["pairs"].sum()) * len(rows)
    t0 = time.perf_counter()
    OA.attention_head(q[0, 0], k[0, 0], v[0, 0], w.mask_kind, window=w.window or None,
                      doc_id=None if doc is None else doc.numpy(), score_kind=w.score_kind,
                      softcap=w.softcap, rows=rows, bitmap=words)
    dt = time.perf_counter() - t0
    credited = sum(4.0 * w.D * 128 * int(fig["per_row"][r // 128]) for r in rows)
    return dt, credited


def max_over_ranks(x: float, device) -> float:
    """The maximum of a per-rank figure over all ranks (a time: the slowest rank
    decides the job's time); the figure itself on one rank."""
    if not torch.distributed.is_available() or not torch.distributed.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def launch_ranks(argv, n: int) -> int:
    """Start this script as n ranks on this node (one process per GPU) through
    torch.distributed.run, rendezvous on 127.0.0.1; returns the launcher's exit code."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={free_port()}",
           os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def init_ranks(backend: str, local: int):
    from datetime import timedelta
    kw = {"timeout": timedelta(seconds=120)}
    if backend == "nccl":
        kw["device_id"] = torch.device("cuda", local)
    torch.distributed.init_process_group(backend, **kw)


def dry_run(args, rank, world):
    """Launcher and timing check without a GPU (gloo, CPU): each rank "steps" for a
    rank-dependent time; the job's time is the maximum over ranks, as in the real
    bench, and rank 0 prints one JSON line."""
    per_step = 0.01 * (rank + 1)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        time.sleep(per_step)
    ms = (time.perf_counter() - t0) * 1e3
    gathered = [None] * world
    if world > 1:
        torch.distributed.all_gather_object(gathered, ms)
    else:
        gathered = [ms]
    job_ms = max_over_ranks(ms, "cpu")
    if rank == 0:
        print(json.dumps({"dry_run": True, "n_gpus": world, "steps": args.steps,
                          "ms_per_step": job_ms / args.steps, "rank_ms": gathered,
                          "value": world * args.steps / (job_ms * 1e-3), "unit": "steps/s"}))


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=W.C3_SWA256_32K.name, choices=sorted(W.BY_NAME))
    ap.add_argument("--cpu-rows", type=int, default=32768,
                    help="oracle rows timed for cpu_baseline (bounded sample)")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (column lists + fa_flex_attention_bwd) of the "
                         "workload instead of the forward step; prints its own JSON line")
    ap.add_argument("--profile", action="store_true",
                    help="short run for profilers: warm-up and timed steps only (no clock "
                         "window, no end-to-end leg, no CPU baseline); not a bench value")
    ap.add_argument("--dry-run", action="store_true",
                    help="launcher and max-over-ranks timing check on CPU (gloo); no GPU")
    args = ap.parse_args()
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: start the ranks here (the driver may start them itself)
        sys.exit(launch_ranks(sys.argv[1:], args.gpus))
    w = W.BY_NAME[args.workload]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but {world} ranks were launched")
    if args.dry_run:
        if world > 1:
            init_ranks("gloo", local)
        dry_run(args, rank, world)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    peaks, peaks_src = load_peaks()
    fig = work_figures(w)

    if args.impl == "reference":
        if rank != 0:
            return
        rows_per_step = 64
        g = np.random.default_rng(0)

        def sample():  # decode: the new queries of the first few heads
            if is_decode(w):
                return np.arange(min(w.H, 8))
            return np.sort(g.integers(0, w.L, rows_per_step))
        for _ in range(args.warmup):
            oracle_sample(w, sample(), fig)
        tot_s, tot_f = 0.0, 0.0
        for _ in range(args.steps):
            dt, fl = oracle_sample(w, sample(), fig)
            tot_s += dt
            tot_f += fl
        value = tot_f / tot_s / 1e12
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                # each step is a bounded sample of the workload (see cpu_baseline.sample):
                # ms_per_step is the time those samples took; the whole workload at this
                # rate would take ms_per_step_extrapolated
                "ms_per_step": tot_s * 1e3 / args.steps,
                "ms_per_step_extrapolated": fig["flops"] / (value * 1e12) * 1e3,
                "sampled_s": tot_s,
                "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {**w.describe(), "parallelism": "none (host cores)"},
                "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(),
                                 "kind": "oracle",
                                 "sample": (f"all new queries of {min(w.H, 8)} heads of batch 0 per step"
                                            if is_decode(w) else
                                            f"{rows_per_step} random query rows of head (0,0) per "
                                            "step") + "; ms_per_step is the sample's time, "
                                                      "ms_per_step_extrapolated the whole "
                                                      "workload's"},
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    if world > 1:
        init_ranks("nccl", local)
    device = torch.device("cuda", local)
    if args.backward:
        run_backward(args, w, world, device, fig)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    r = run_ours(args, w, rank, world, device)

    total_flops = fig["flops"] * args.steps * world
    value = total_flops / (r["total_ms"] * 1e-3) / 1e12
    fwd_avg = statistics.mean(r["fwd_ms"])
    fwd_med = statistics.median(r["fwd_ms"])
    fwd_tflops = fig["flops"] / (fwd_avg * 1e-3) / 1e12
    fwd_gbs = fig["bytes"] / (fwd_avg * 1e-3) / 1e9
    hbm_peak = peaks["hbm_gbs"]
    tc_peak = peaks["bf16_tflops"]
    e2e_value = fig["flops"] * args.steps * world / (r["e2e"]["ms"] * 1e-3) / 1e12
    tensor_frac = fwd_tflops / tc_peak
    hbm_frac = fwd_gbs / hbm_peak
    bound = "hbm" if hbm_frac >= tensor_frac else "tensor"
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": fwd_gbs, "peak": hbm_peak, "unit": "GB/s",
                "frac": hbm_frac, "traffic": ncu_traffic(w)}
    else:
        roof = {"bound": "tensor", "achieved": fwd_tflops, "peak": tc_peak, "unit": "TFLOP/s",
                "frac": tensor_frac, "traffic": ncu_traffic(w)}
    roof["peak_source"] = f"{peaks_src} (MEASURED_PEAKS.json)" if peaks_src == "measured" else "fallback"
    if is_decode(w):
        roof["kernel"] = "decode_mma_kernel + decode_combine_kernel (fa_flex_attention_decode)"
    else:
        roof["kernel"] = "fwd_kernel (fa_flex_attention_fwd)"
    page_ms = PAGE_FWD_MS.get(w.name)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": r["total_ms"] / args.steps,
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": (value / (fig["flops"] / (page_ms * 1e-3) / 1e12)) if page_ms else None,
            "dtype": w.dtype_name, "data": "synthetic",
            "config": {**w.describe(), "parallelism": f"replicas x{world}" if world > 1 else "none",
                       "l2": "flushed between timed steps (512 MiB write, untimed)",
                       "step": ("fa_flex_attention_decode" if is_decode(w)
                                else "fa_create_block_mask + fa_flex_attention_fwd")},
            "fwd_ms": fwd_avg, "fwd_ms_median": fwd_med, "fwd_tflops": fwd_tflops,
            "fwd_tensor_frac": tensor_frac, "fwd_hbm_gbs": fwd_gbs, "fwd_hbm_frac": hbm_frac,
            "mask_build_ms": statistics.mean(r["mask_ms"]),
            "live_blocks_per_head": fig["live_blocks"], "live_gflop": fig["flops"] / 1e9,
            **({"step_kind": "decode (split-KV forward + merge; no mask tables)"}
               if is_decode(w) else {}),
            "algorithmic_mb": fig["bytes"] / 1e6,
            "roofline": roof,
            # this library's launches per timed step: decode = chunk kernel + merge;
            # causal / window masks = one table launch + the forward; documents and
            # tabulated masks = classify + order + the forward
            "gpu_launches": (2 if is_decode(w) or w.mask_kind in (W.MASK_CAUSAL,
                                                                   W.MASK_SLIDING_WINDOW_CAUSAL)
                             else 3) * args.steps,
            "clocks": r["clocks"],
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": r["e2e"]["h2d"],
                    "d2h_bytes_per_step": r["e2e"]["d2h"],
                    "ms_per_step": r["e2e"]["ms"] / args.steps}}
    if rank == 0 and world == 1 and not args.profile:
        if is_decode(w):  # the oracle on all new queries of every head of batch 0
            rows = np.arange(w.H)
        else:
            rows = np.sort(np.random.default_rng(1).choice(w.L, size=min(args.cpu_rows, w.L),
                                                           replace=False))
        dt, credited = oracle_sample(w, rows, fig)
        line["cpu_baseline"] = {"value": credited / dt / 1e12, "unit": UNIT, "cores": cpu_threads(),
                                "kind": "oracle",
                                "sample": (f"all {w.L} new queries of the {len(rows)} heads of "
                                           f"batch 0, {dt:.1f} s; visible-pair FLOPs credited"
                                           if is_decode(w) else
                                           f"{len(rows)} random query rows of head (0,0), "
                                           f"{dt:.1f} s; live-block FLOPs of those rows credited")}
    if world == 1 and not args.profile and args.workload == W.C3_SWA256_32K.name:
        # the other configurations of the benchmark set, forward kernel only, same run
        line["configs"] = config_sweep(device)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))


if __name__ == "__main__":
    main()
