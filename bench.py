#!/usr/bin/env python
"""Benchmark of the block-sparse attention hot path on B200.

One step is one pass of the whole path over one batch of synthetic input:
  1. bsattn_build_index   causal 256 x 256 block mask -> CSR and the
                          longest-first row order             (4 small launches)
  2. bsattn_fwd_prefill   BLASST prefill, B1 Hq32/Hkv8 N32768 d128, causal,
                          tiles 128, lambda = a / N                (1 launch)
  3. bsattn_fwd_decode    BLASST split-KV decode, B64 Hq32/Hkv8 L131072 d128,
                          tiles 128, 16 splits, lambda = a / L      (2 launches)
Each phase is timed with CUDA events on the launching stream.  The headline
`value` is prefill TFLOP/s over the tiles the kernel really processed
(2*128*128*128 flops per visited tile for Q K^T plus the same per executed
tile for P V); the `decode` object carries decode GB/s over the bytes the
kernel must read (Q, O, every visited K tile, every executed V tile).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--a 10] [--impl native|reference]

Under torchrun every rank runs the same per-GPU workload on its own seeded
inputs (weak scaling: (batch, head) units are independent, no collective on
the data path); times are the max over ranks and `value` aggregates all ranks.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same
workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "block-sparse attn TFLOP/s (executed tiles) & decode GB/s, % of B200 peak"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
BLK = 128
D = 128
TILE_FLOP = 2 * BLK * BLK * D          # one 128x128x128 GEMM tile


def log(*a):
    if int(os.environ.get("RANK", "0")) == 0:
        print(*a, file=sys.stderr, flush=True)


def profiled_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu capture
    (profiles/traffic.json), or None when the kernel's sources changed since
    the counters were taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        t = json.load(f).get(kernel)
    if not t:
        return None
    h = hashlib.sha256()
    for src in t["sources"]:
        with open(os.path.join(ROOT, src), "rb") as f:
            h.update(f.read())
    return t["traffic_bytes_per_launch"] if h.hexdigest()[:16] == t["sources_sha256_16"] else None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------------ workloads
def make_inputs(rank: int, a: float):
    from block_sparse_attention_bsattn_b200 import inputs
    ps, ds = rank_seeds(rank)
    pw = inputs.workload("blasst_prefill", device="cuda", seed=ps)
    dw = inputs.workload("blasst_decode", device="cuda", seed=ds)
    mask = torch.ones(1, pw.nq, pw.nk, dtype=torch.uint8, device="cuda")
    return pw, dw, mask


class Step:
    """Preallocated buffers and one pass of the path."""

    def __init__(self, pw, dw, mask, a):
        from block_sparse_attention_bsattn_b200 import inputs, ops
        self.ops = ops
        self.pw, self.dw, self.mask = pw, dw, mask
        self.opts = {"reverse": False, "skip_v": False, "sink_seed": False, "seq_lens": None}
        self.set_a(a)
        nb = pw.nq
        self.row_ptr = torch.empty(nb + 1, dtype=torch.int32, device="cuda")
        self.col_idx = torch.empty(nb * nb, dtype=torch.int32, device="cuda")
        self.nnz = torch.empty(1, dtype=torch.int32, device="cuda")
        self.row_order = torch.empty(nb, dtype=torch.int32, device="cuda")
        self.o = torch.empty_like(pw.q)
        self.lse = torch.empty(pw.B, pw.Hq, pw.N, dtype=torch.float32, device="cuda")
        self.do = torch.empty_like(dw.q)
        self.dlse = torch.empty(dw.B, dw.Hq, dtype=torch.float32, device="cuda")
        ws = ops.bsattn_decode_workspace_size(dw.B, dw.Hq, dw.d, dw.num_splits)
        self.ws = torch.empty(ws, dtype=torch.uint8, device="cuda")
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        self._inputs = inputs

    def set_a(self, a):
        from block_sparse_attention_bsattn_b200 import inputs
        self.a = a
        self.p_lam = inputs.lambda_for(a, self.pw.N)
        self.d_lam = inputs.lambda_for(a, self.dw.N)

    def index(self):
        lib = self.ops._lib
        rc = lib.bsattn_build_index(self.ops._ptr(self.mask), 1, self.pw.nq, self.pw.nk, BLK, BLK, 1,
                                    self.ops._ptr(self.row_ptr), self.ops._ptr(self.col_idx),
                                    self.col_idx.numel(), self.ops._ptr(self.nnz),
                                    self.ops._ptr(self.row_order), self.ops._ptr(self.status),
                                    self.ops._stream(None))
        assert rc == 0

    def prefill(self, tile_status=None):
        pw = self.pw
        self.ops.bsattn_fwd_prefill(pw.q, pw.k, pw.v, BLK, pw.scale, True, self.p_lam,
                                    self.row_ptr, self.col_idx, 1, o=self.o, lse=self.lse,
                                    tile_status=tile_status, status=self.status,
                                    row_order=self.row_order, reverse=self.opts["reverse"],
                                    skip_v=self.opts["skip_v"])

    def decode(self, tile_status=None):
        dw = self.dw
        self.ops.bsattn_fwd_decode(dw.q, dw.k, dw.v, BLK, dw.num_splits, dw.scale, self.d_lam,
                                   o=self.do, lse=self.dlse, workspace=self.ws,
                                   tile_status=tile_status, status=self.status,
                                   sink_seed=self.opts["sink_seed"], seq_lens=self.opts["seq_lens"])

    LAUNCHES = 4 + 1 + 2

    def counts(self):
        """Visited / executed tiles of this input (decisions are deterministic)."""
        pw, dw = self.pw, self.dw
        self.index()
        pst = torch.zeros(pw.B, pw.Hq, pw.nq, pw.nk, dtype=torch.uint8, device="cuda")
        self.prefill(pst)
        T = -(-dw.N // BLK)
        dst = torch.zeros(dw.B, dw.Hkv, T, dtype=torch.uint8, device="cuda")
        self.decode(dst)
        torch.cuda.synchronize()
        assert self.status.item() == 0, self.ops.bsattn_status_string(self.status.item())
        pv, pe = int((pst > 0).sum()), int((pst == 2).sum())
        dv, de = int((dst > 0).sum()), int((dst == 2).sum())
        return {"p_visited": pv, "p_executed": pe, "d_visited": dv, "d_executed": de}


def prefill_flops(c):
    return TILE_FLOP * (c["p_visited"] + c["p_executed"])


def decode_bytes(dw, c):
    tile_bytes = BLK * dw.d * 2
    return 2 * dw.B * dw.Hq * dw.d * 2 + tile_bytes * (c["d_visited"] + c["d_executed"])


def timed_phases(step: Step, steps: int, phases=("index", "prefill", "decode")):
    """Run `steps` steps; returns per-phase total ms and the whole region ms."""
    stream = torch.cuda.current_stream()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(phases) + 1)]
          for _ in range(steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for s in range(steps):
        ev[s][0].record(stream)
        for i, ph in enumerate(phases):
            getattr(step, ph)()
            ev[s][i + 1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    per = {ph: sum(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(steps))
           for i, ph in enumerate(phases)}
    return per, t0.elapsed_time(t1)


def _reduce_device():
    return "cuda" if dist.get_backend() == "nccl" else "cpu"


def max_over_ranks(x: float) -> float:
    """Largest value over all ranks (times: the slowest rank sets the step)."""
    if dist.is_initialized():
        t = torch.tensor([x], dtype=torch.float64, device=_reduce_device())
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return x


def sum_over_ranks(x: float) -> float:
    """Sum over all ranks (work: every rank processes its own units)."""
    if dist.is_initialized():
        t = torch.tensor([x], dtype=torch.float64, device=_reduce_device())
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
        return float(t.item())
    return x


def rank_seeds(rank: int):
    """Seeds of the prefill and decode inputs of one rank: each rank draws its
    own batch of the same workload (weak scaling)."""
    return 1237 + 1000 * rank, 1238 + 1000 * rank


def whole_job_rate(units_this_rank: float, ms_this_rank: float) -> float:
    """Units per second of the whole job: all ranks' units over the slowest
    rank's time."""
    return sum_over_ranks(units_this_rank) / (max_over_ranks(ms_this_rank) * 1e-3)


def barrier():
    if dist.is_initialized():
        dist.barrier()


# ------------------------------------------------------------------ e2e
def e2e_run(step: Step, steps: int):
    """Prefill through host buffers: the block mask copied in and indexed,
    then pinned Q/K/V in, prefill and O out per KV head with the copies
    overlapped (bsattn_fwd_prefill_host); decode with its KV cache resident:
    the query copied in, O copied out.  Copies are inside the timed region."""
    pw, dw = step.pw, step.dw
    hq = pw.q.cpu().pin_memory()
    hk = pw.k.cpu().pin_memory()
    hv = pw.v.cpu().pin_memory()
    hm = step.mask.cpu().pin_memory()
    ho = torch.empty(pw.q.shape, dtype=pw.q.dtype).pin_memory()
    hdq = dw.q.cpu().pin_memory()
    hdo = torch.empty(dw.q.shape, dtype=dw.q.dtype).pin_memory()
    stream = torch.cuda.current_stream()

    ops = step.ops

    def one(s_ev):
        s_ev[0].record(stream)
        step.mask.copy_(hm, non_blocking=True)
        step.index()
        # Q/K/V in, prefill, O out per KV head, the copies overlapped with the
        # kernels of other KV heads (bsattn_fwd_prefill_host)
        ops.bsattn_fwd_prefill_host(hq, hk, hv, ho, pw.q, pw.k, pw.v, step.o, BLK, pw.scale,
                                    True, step.p_lam, step.row_ptr, step.col_idx, 1,
                                    row_order=step.row_order, kv_heads_per_chunk=1,
                                    status=step.status)
        s_ev[1].record(stream)
        dw.q.copy_(hdq, non_blocking=True)
        step.decode()
        hdo.copy_(step.do, non_blocking=True)
        s_ev[2].record(stream)

    for _ in range(2):
        one([torch.cuda.Event(enable_timing=True) for _ in range(3)])
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    barrier()
    torch.cuda.synchronize()
    for s in range(steps):
        one(evs[s])
    torch.cuda.synchronize()
    barrier()
    p_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    d_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    h2d_p = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hm))
    d2h_p = ho.numel() * ho.element_size()
    h2d_d = hdq.numel() * hdq.element_size()
    d2h_d = hdo.numel() * hdo.element_size()
    return p_ms, d_ms, (h2d_p, d2h_p, h2d_d, d2h_d)


# ------------------------------------------------------------------ CPU baseline (oracle)
def oracle_prefill_sample(pw, a, n_items, seed=0):
    """Time the fp64 oracle on n_items query tiles of the prefill workload
    (spread over the causal triangle); returns (TFLOP/s counted as on the GPU,
    seconds, threads, sample description)."""
    import oracle
    from block_sparse_attention_bsattn_b200 import inputs
    rng = np.random.default_rng(seed)
    items = sorted({(0, int(rng.integers(pw.Hq)), int(i))
                    for i in np.linspace(0, pw.nq - 1, n_items).astype(int)})
    q, k, v = pw.q.cpu(), pw.k.cpu(), pw.v.cpu()
    lam = inputs.lambda_for(a, pw.N)
    t = time.perf_counter()
    r = oracle.prefill(q, k, v, pw.block, pw.scale, True, lam, items=items)
    dt = time.perf_counter() - t
    st = r["status"]
    flops = TILE_FLOP * (int((st > 0).sum()) + int((st == 2).sum()))
    return flops / dt / 1e12, dt, oracle.num_threads(), \
        f"{len(items)} query tiles of {pw.B * pw.Hq * pw.nq} (all their visited tiles), a={a}"


def oracle_decode_sample(dw, a, n_pairs, seed=0):
    import oracle
    from block_sparse_attention_bsattn_b200 import inputs
    rng = np.random.default_rng(seed)
    pairs = sorted({(int(rng.integers(dw.B)), int(rng.integers(dw.Hkv))) for _ in range(n_pairs)})
    qs, ks, vs = oracle.decode_problems(dw.q, dw.k, dw.v, pairs)
    qs, ks, vs = qs.cpu(), ks.cpu(), vs.cpu()
    lam = inputs.lambda_for(a, dw.N)
    t = time.perf_counter()
    r = oracle.decode(qs, ks, vs, dw.block, dw.scale, lam, dw.num_splits)
    dt = time.perf_counter() - t
    st = r["status"]
    g = dw.Hq // dw.Hkv
    byt = len(pairs) * 2 * g * dw.d * 2 + BLK * dw.d * 2 * (int((st > 0).sum()) + int((st == 2).sum()))
    return byt / dt / 1e9, dt, oracle.num_threads(), \
        f"{len(pairs)} (batch, kv-head) problems of {dw.B * dw.Hkv}, a={a}"


# ------------------------------------------------------------------ static masks
STATIC_WORKLOADS = ("tiny", "mmdit", "videodit")
L2_FLUSH_BYTES = 256 << 20     # more than the 126 MB L2


def time_calls(fn, n, flush=None):
    """Mean CUDA-event time (ms) of fn over n calls on the current stream;
    `flush` (writing a buffer larger than L2) runs between calls, outside the
    events."""
    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    for a, b in evs:
        if flush is not None:
            flush()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs) / n


def static_kernel_name(w):
    """The kernel bsattn_fwd_prefill dispatches a block mask with one query
    head per KV head to: one query tile per CTA."""
    return f"prefill_kernel<{w.d}, {w.block}, 0>"


def static_section(iters, warmup, peak):
    """The static-mask workloads at full size (lambda = 0): tiny (B1 H2 N512 d64,
    block 64), multimodal DiT (B1 H24 N4352 d64) and Video-DiT (B1 H16 N66048
    d128), each timed with CUDA events with L2 flushed between calls, and the
    same kernel with an all-ones mask as the dense comparison (the DiT page,
    section 4.2: kept-block fraction against runtime).  TFLOP/s count
    4 * block^2 * d per executed tile (Q K^T and P V)."""
    from block_sparse_attention_bsattn_b200 import inputs, ops
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    flush = lambda: flush_buf.fill_(1)   # noqa: E731
    out = {}
    for name in STATIC_WORKLOADS:
        w = inputs.workload(name, device="cuda")
        o = torch.empty_like(w.q)
        res = {"workload": f"{name} B{w.B} H{w.Hq} N{w.N} d{w.d} block{w.block}, non-causal, "
                           f"lambda=0", "kernel": static_kernel_name(w)}
        for which, m in (("mask", w.mask.cuda()), ("dense", torch.ones_like(w.mask).cuda())):
            rp, ci, nnz, order = ops.bsattn_build_index(m, w.block, w.block, False,
                                                        with_order=True)
            tiles = int(nnz.sum()) * w.B * w.Hq
            fn = lambda: ops.bsattn_fwd_prefill(w.q, w.k, w.v, w.block, w.scale, False, 0.0,  # noqa: E731
                                                rp, ci, 1, o=o, want_lse=False, row_order=order)
            for _ in range(warmup):
                fn()
            torch.cuda.synchronize()
            ms = max_over_ranks(time_calls(fn, iters, flush))
            flops = 4 * w.block * w.block * w.d * tiles
            tf = flops / (ms * 1e-3) / 1e12
            if which == "mask":
                res.update(tiles_executed=tiles, ms=ms, tflops=tf, frac=tf / peak,
                           flops_per_launch=flops)
            else:
                res.update(dense_tiles=tiles, dense_ms=ms, dense_tflops=tf)
        res["kept_frac"] = res["tiles_executed"] / res["dense_tiles"]
        res["time_vs_dense"] = res["ms"] / res["dense_ms"]
        out[name] = res
        del w, o
        torch.cuda.empty_cache()
    del flush_buf
    torch.cuda.empty_cache()
    return out


def decode_operating_point(dw, iters, warmup):
    """The BLASST page's decode operating point (73.2% of the decode's tiles
    skipped): on this recipe 4 splits at a = 160, fixed by an oracle sweep
    (tests/golden/decode_operating_point.txt); timed against the same kernel
    with lambda = 0 and the same splits."""
    from block_sparse_attention_bsattn_b200 import inputs, ops
    splits, a = inputs.DECODE_OP_SPLITS, inputs.DECODE_OP_A
    T = -(-dw.N // BLK)
    ws = torch.empty(ops.bsattn_decode_workspace_size(dw.B, dw.Hq, dw.d, splits),
                     dtype=torch.uint8, device="cuda")
    o = torch.empty_like(dw.q)
    res = {"num_splits": splits, "a": a, "pages": "1.48x over FlashAttention-3 at 73.2% "
                                                "sparsity (H200/B200; context, not the target)"}
    for which, aa in (("sparse", a), ("dense", 0.0)):
        lam = inputs.lambda_for(aa, dw.N)
        st = torch.zeros(dw.B, dw.Hkv, T, dtype=torch.uint8, device="cuda")
        ops.bsattn_fwd_decode(dw.q, dw.k, dw.v, BLK, splits, dw.scale, lam, o=o, want_lse=False,
                              workspace=ws, tile_status=st)
        torch.cuda.synchronize()
        vis, exe = int((st > 0).sum()), int((st == 2).sum())
        fn = lambda: ops.bsattn_fwd_decode(dw.q, dw.k, dw.v, BLK, splits, dw.scale, lam, o=o,  # noqa: E731
                                           want_lse=False, workspace=ws)
        for _ in range(warmup):
            fn()
        ms = max_over_ranks(time_calls(fn, iters))
        byt = 2 * dw.B * dw.Hq * dw.d * 2 + BLK * dw.d * 2 * (vis + exe)
        if which == "sparse":
            res.update(ms=ms, gbs=byt / (ms * 1e-3) / 1e9, skipped_frac=1 - exe / vis)
        else:
            res.update(dense_ms=ms, dense_gbs=byt / (ms * 1e-3) / 1e9)
    res["speedup_vs_dense"] = res["dense_ms"] / res["ms"]
    return res


def oracle_per_config(pw, dw, a):
    """The fp64 oracle on the host cores, one bounded sample per workload:
    tiny and multimodal DiT in full, Video-DiT and the BLASST prefill on one
    head (all its query tiles), the BLASST decode on 8 (sequence, KV head)
    problems.  Each entry: seconds, tiles per second, the throughput counted
    as on the GPU, and the full workload's time extrapolated by its number
    of (sequence, head) units."""
    import oracle
    from block_sparse_attention_bsattn_b200 import inputs
    out = {}
    for name, heads in (("tiny", None), ("mmdit", None), ("videodit", 1)):
        w = inputs.workload(name, generate=False)
        h = w.Hq if heads is None else heads
        q, k, v = inputs.normal_qkv(w.B, h, h, w.N, w.d, "cpu", 1234 + len(name))
        t = time.perf_counter()
        r = oracle.prefill(q, k, v, w.block, w.scale, False, 0.0, mask=w.mask.numpy())
        dt = time.perf_counter() - t
        tiles = int((r["status"] == 2).sum())
        flops = 4 * w.block * w.block * w.d * tiles
        out[name] = {"seconds": dt, "tiles_per_s": tiles / dt, "tflops": flops / dt / 1e12,
                     "sample": f"{h} of {w.Hq} heads, all query tiles ({tiles} tiles)",
                     "extrapolated_full_s": dt * w.Hq / h}
    # BLASST prefill: query head 0 and its KV head, every query tile
    q, k, v = pw.q[:, :1].cpu(), pw.k[:, :1].cpu(), pw.v[:, :1].cpu()
    t = time.perf_counter()
    r = oracle.prefill(q, k, v, pw.block, pw.scale, True, inputs.lambda_for(a, pw.N))
    dt = time.perf_counter() - t
    st = r["status"]
    vis, exe = int((st > 0).sum()), int((st == 2).sum())
    out["blasst_prefill"] = {"seconds": dt, "tiles_per_s": vis / dt,
                             "tflops": TILE_FLOP * (vis + exe) / dt / 1e12,
                             "sample": f"1 of {pw.Hq} query heads, all query tiles "
                                       f"({vis} visited, {exe} executed), a={a:g}",
                             "extrapolated_full_s": dt * pw.Hq}
    gb, ddt, _, dsample = oracle_decode_sample(dw, a, 8)
    out["blasst_decode"] = {"seconds": ddt, "gbs": gb, "sample": dsample,
                            "extrapolated_full_s": ddt * dw.B * dw.Hkv / 8}
    return out


def backward_section(step, iters, warmup, peak):
    """Gradients of the step's BLASST prefill (same inputs, same a) with its
    executed tiles held fixed (bsattn_bwd_prefill: a row kernel, dK/dV, dQ).
    Work: 5 GEMM tiles of 2*128^3 flops per executed tile (S, dP, dV, dK, dQ;
    the kernels issue 7, recomputing S and dP for dQ)."""
    from block_sparse_attention_bsattn_b200 import ops
    pw = step.pw
    st = torch.zeros(pw.B, pw.Hq, pw.nq, pw.nk, dtype=torch.uint8, device="cuda")
    step.index()
    step.prefill(st)
    g = torch.Generator(device="cuda").manual_seed(4242)
    dout = torch.randn(pw.q.shape, generator=g, device="cuda").to(torch.bfloat16)
    dq, dk, dv = torch.empty_like(pw.q), torch.empty_like(pw.k), torch.empty_like(pw.v)
    ws = torch.empty(ops.bsattn_bwd_prefill_workspace_size(pw.B, pw.Hq, pw.N, BLK),
                     dtype=torch.uint8, device="cuda")
    fn = lambda: ops.bsattn_bwd_prefill(pw.q, pw.k, pw.v, step.o, dout, step.lse, st, BLK,  # noqa: E731
                                        pw.scale, True, status=step.status, dq=dq, dk=dk, dv=dv,
                                        workspace=ws)
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ms = max_over_ranks(time_calls(fn, iters))
    exe = int((st == 2).sum())
    flops = 5 * TILE_FLOP * exe
    tf = flops / (ms * 1e-3) / 1e12
    return {"kernels": "bwd_rows_kernel + bwd_dkdv_kernel<128> + bwd_dq_kernel<128>",
            "ms": ms, "tflops": tf, "frac": tf / peak, "flops_per_call": flops,
            "issued_tflops": 7 * TILE_FLOP * exe / (ms * 1e-3) / 1e12,
            "executed_tiles": exe, "a": step.a}


# ------------------------------------------------------------------ main
def config_dict(pw, dw, a, n):
    return {
        "workload": f"blasst_prefill B{pw.B} Hq{pw.Hq}/Hkv{pw.Hkv} N{pw.N} d{pw.d} causal tile{BLK} "
                    f"+ blasst_decode B{dw.B} Hq{dw.Hq}/Hkv{dw.Hkv} L{dw.N} d{dw.d} tile{BLK} "
                    f"splits{dw.num_splits}, a={a:g} (lambda=a/L)",
        "prefill": {"B": pw.B, "Hq": pw.Hq, "Hkv": pw.Hkv, "N": pw.N, "d": pw.d, "tile": BLK,
                    "causal": True, "index": "causal 256x256 block mask -> CSR each step"},
        "decode": {"B": dw.B, "Hq": dw.Hq, "Hkv": dw.Hkv, "L": dw.N, "d": dw.d, "tile": BLK,
                   "num_splits": dw.num_splits},
        "a": a,
        "l2": "no flush: inputs larger than L2 (prefill Q+K+V 384 MiB, decode K+V 32 GiB)",
        "parallelism": f"dp{n}: independent (batch, head) units per rank, no collective",
    }


def run_reference(args):
    """Oracle on the host cores, same metric/config, bounded sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.build()
    from block_sparse_attention_bsattn_b200 import inputs
    pw = inputs.workload("blasst_prefill", device="cpu")
    dw_shape = inputs.workload("blasst_decode", generate=False)
    # decode problems are independent (batch, kv-head) pairs: draw a few with the
    # same recipe and shapes instead of materialising the 32 GiB cache on the host
    q, k, v = inputs.blasst_decode_qkv(2, dw_shape.Hq, dw_shape.Hkv, dw_shape.N, dw_shape.d, "cpu",
                                       1238)
    dw_shape.B = 2
    dw_shape.q, dw_shape.k, dw_shape.v = q, k, v
    times, vals, dvals = [], [], []
    n_items = 4
    for s in range(args.warmup + args.steps):
        tf, dt, cores, sample = oracle_prefill_sample(pw, args.a, n_items, seed=s)
        gb, ddt, _, dsample = oracle_decode_sample(dw_shape, args.a, 1, seed=s)
        if s >= args.warmup:
            times.append((dt + ddt) * 1e3)
            vals.append(tf)
            dvals.append(gb)
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 0,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(pw, inputs.workload("blasst_decode", generate=False),
                                                   args.a, 1),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"per step: {sample}; decode {dsample}"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "decode": {"value": statistics.mean(dvals), "unit": "GB/s"},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--a", type=float, default=10.0)
    ap.add_argument("--impl", choices=("native", "reference"), default="native")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-variants", action="store_true")
    ap.add_argument("--no-static", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        run_reference(args)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    peaks, peak_src = load_peaks()

    log("generating inputs ...")
    pw, dw, mask = make_inputs(rank, args.a)
    step = Step(pw, dw, mask, args.a)
    counts = step.counts()
    p_flops = prefill_flops(counts)
    d_bytes = decode_bytes(dw, counts)

    for _ in range(args.warmup):
        step.index(); step.prefill(); step.decode()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.2)
    per, total_ms = timed_phases(step, args.steps)
    barrier()
    clk = clocks.stop()
    total_ms = max_over_ranks(total_ms)
    per = {k: max_over_ranks(v) for k, v in per.items()}
    assert step.status.item() == 0

    K = args.steps
    p_ms = per["prefill"] / K
    d_ms = per["decode"] / K
    i_ms = per["index"] / K
    tf_rank = p_flops / (p_ms * 1e-3) / 1e12
    gb_rank = d_bytes / (d_ms * 1e-3) / 1e9
    value = sum_over_ranks(p_flops) / (p_ms * 1e-3) / 1e12
    d_value = sum_over_ranks(d_bytes) / (d_ms * 1e-3) / 1e9
    strict_flops = 2 * TILE_FLOP * counts["p_executed"]

    # dense comparison and the a-sweep (same kernels, lambda = a / L)
    sweep = []
    if not args.no_sweep:
        for a in (0.0, 1.0, 10.0, 100.0):
            step.set_a(a)
            c = step.counts()
            for _ in range(2):
                step.index(); step.prefill(); step.decode()
            sp, _ = timed_phases(step, max(3, K // 4))
            n = max(3, K // 4)
            sweep.append({
                "a": a,
                "prefill_ms": max_over_ranks(sp["prefill"]) / n,
                "prefill_tflops": prefill_flops(c) / (max_over_ranks(sp["prefill"]) / n * 1e-3) / 1e12,
                "prefill_skipped_frac": 1 - c["p_executed"] / c["p_visited"],
                "decode_ms": max_over_ranks(sp["decode"]) / n,
                "decode_gbs": decode_bytes(dw, c) / (max_over_ranks(sp["decode"]) / n * 1e-3) / 1e9,
                "decode_skipped_frac": 1 - c["d_executed"] / c["d_visited"],
            })
        step.set_a(args.a)

    # the options of the _ex entry points at the same a: descending visit
    # order and V skipping (prefill), sink-seeded splits (decode)
    variants = {}
    if not args.no_variants:
        # cache lengths drawn uniformly from [L/8, L] (seeded): key padding
        g = torch.Generator().manual_seed(4321 + rank)
        varlen = torch.randint(dw.N // 8, dw.N + 1, (dw.B,), generator=g, dtype=torch.int32).cuda()
        for name, opt, phase in (("prefill_reverse", "reverse", "prefill"),
                                 ("prefill_skip_v", "skip_v", "prefill"),
                                 ("decode_sink_seed", "sink_seed", "decode"),
                                 ("decode_varlen", "seq_lens", "decode")):
            step.opts[opt] = varlen if opt == "seq_lens" else True
            c = step.counts()
            for _ in range(2):
                step.index(); getattr(step, phase)()
            n = max(3, K // 4)
            sp, _ = timed_phases(step, n, ("index", phase))
            ms = max_over_ranks(sp[phase]) / n
            if phase == "prefill":
                variants[name] = {"ms": ms, "tflops": prefill_flops(c) / (ms * 1e-3) / 1e12,
                                  "skipped_frac": 1 - c["p_executed"] / c["p_visited"],
                                  "vs_default_ms": p_ms}
            else:
                variants[name] = {"ms": ms, "gbs": decode_bytes(dw, c) / (ms * 1e-3) / 1e9,
                                  "skipped_frac": 1 - c["d_executed"] / c["d_visited"],
                                  "vs_default_ms": d_ms,
                                  "note": "bytes exclude the one extra K tile per split read "
                                          "to seed the running max" if opt == "sink_seed" else
                                          "cache lengths uniform in [L/8, L]; bytes count the "
                                          "valid tiles only"}
            step.opts[opt] = None if opt == "seq_lens" else False
        variants["decode_operating_point"] = decode_operating_point(dw, max(3, K // 4), 2)

    e2e = None
    if not args.no_e2e:
        e_p_ms, e_d_ms, byts = e2e_run(step, max(3, K // 2))
        n = max(3, K // 2)
        e_p_ms = max_over_ranks(e_p_ms) / n
        e_d_ms = max_over_ranks(e_d_ms) / n
        e2e = {"value": sum_over_ranks(p_flops) / (e_p_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": byts[0], "d2h_bytes_per_step": byts[1],
               "ms_per_step": e_p_ms,
               "decode": {"value": sum_over_ranks(d_bytes) / (e_d_ms * 1e-3) / 1e9, "unit": "GB/s",
                          "ms_per_step": e_d_ms, "h2d_bytes_per_step": byts[2],
                          "d2h_bytes_per_step": byts[3],
                          "note": "KV cache resident on the device; the query and O cross PCIe"}}

    bwd = None
    if not args.no_backward:
        bwd = backward_section(step, max(3, K // 4), 2, peaks["bf16_tflops"])
        assert step.status.item() == 0

    static = None
    if not args.no_static:
        clocks_s = ClockSampler(local)
        clocks_s.start()
        static = static_section(max(5, K // 2), 3, peaks["bf16_tflops"])
        static["clocks"] = clocks_s.stop()
        static["peak"] = {"bf16_tflops": peaks["bf16_tflops"],
                          "source": f"{peak_src} bf16 burst (cuBLAS)"}
        static["l2"] = "flushed between calls (a 256 MiB write outside the timed events)"

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        per = oracle_per_config(pw, dw, args.a)
        c4 = per["blasst_prefill"]
        cpu = {"value": c4["tflops"], "unit": "TFLOP/s", "cores": oracle.num_threads(),
               "kind": "oracle", "sample": f"blasst_prefill: {c4['sample']}; "
                                           f"{c4['seconds']:.1f} s",
               "decode": {"value": per["blasst_decode"]["gbs"], "unit": "GB/s",
                          "sample": f"{per['blasst_decode']['sample']}; "
                                    f"{per['blasst_decode']['seconds']:.1f} s"},
               "per_config": per,
               "note": "a baseline, not the target: the plain fp64 oracle as it stands"}

    bf16_peak = peaks["bf16_tflops"]
    hbm_peak = peaks["hbm_gbs"]
    prefill_roof = {"kernel": "prefill_pair_kernel<128, 0, %d> (two GQA heads per CTA%s)"
                              % (int(args.a > 0), ", skip vote" if args.a > 0 else ""),
                    "bound": "tensor", "achieved": tf_rank, "peak": bf16_peak,
                    "unit": "TFLOP/s", "frac": tf_rank / bf16_peak,
                    "traffic": profiled_traffic("prefill_pair_kernel<128, 0, %d>" % int(args.a > 0)),
                    "peak_source": f"{peak_src} bf16 burst (cuBLAS)",
                    "flops_per_launch": p_flops,
                    "strict_flops_per_launch": strict_flops,
                    "strict_tflops": strict_flops / (p_ms * 1e-3) / 1e12,
                    "launch_ms": p_ms,
                    # context only: the step runs long enough for the board's
                    # power cap to lower the SM clock, which the burst peak
                    # does not see; cuBLAS under the same cap sustains this
                    "frac_of_sustained_peak": tf_rank / peaks["bf16_tflops_sustained"],
                    "sustained_peak": peaks["bf16_tflops_sustained"]}
    decode_roof = {"kernel": "decode_tc_kernel<128, 4, 128> + decode_combine_kernel",
                   "bound": "hbm", "achieved": gb_rank, "peak": hbm_peak,
                   "unit": "GB/s", "frac": gb_rank / hbm_peak,
                   "traffic": profiled_traffic("decode_tc_kernel<128, 4, 128>"),
                   "peak_source": f"{peak_src} copy bandwidth",
                   "bytes_per_launch": d_bytes, "launch_ms": d_ms}
    # the top-level roofline is the one of the kernel that takes the larger
    # share of the step; the other is reported beside it
    dominant = "decode" if d_ms > p_ms else "prefill"
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": total_ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": config_dict(pw, dw, args.a, world),
        "roofline": dict(decode_roof if dominant == "decode" else prefill_roof,
                         dominant_kernel_of_step=dominant),
        "prefill": {"value": value, "unit": "TFLOP/s", "ms_per_step": p_ms,
                    "roofline": prefill_roof},
        "decode": {"value": d_value, "unit": "GB/s", "ms_per_step": d_ms,
                   "roofline": decode_roof},
        "index_ms_per_step": i_ms,
        "tiles": counts,
        "sparsity": {"prefill_skipped_frac": 1 - counts["p_executed"] / counts["p_visited"],
                     "decode_skipped_frac": 1 - counts["d_executed"] / counts["d_visited"]},
        "sweep": sweep,
        "variants": variants,
        "static": static,
        "backward": bwd,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": Step.LAUNCHES * K,
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
