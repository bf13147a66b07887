"""Time one entry point of the library on a chosen slice of a workload.

    python -m block_sparse_attention_bsattn_b200.microbench prefill --heads 8 --n 8192 --a 10
    python -m block_sparse_attention_bsattn_b200.microbench decode --batch 8 --a 10
    python -m block_sparse_attention_bsattn_b200.microbench videodit --heads 4
    python -m block_sparse_attention_bsattn_b200.microbench table4
    python -m block_sparse_attention_bsattn_b200.microbench backward --heads 32 --a 10

    python -m block_sparse_attention_bsattn_b200.microbench sustained

`sustained` runs the benchmark's two workloads (the 32-head BLASST prefill
through a CSR index with its row order, and the 64-sequence decode) back to
back for about a second per phase -- prefill alone, the index + prefill +
decode step, the step with an idle gap, decode alone -- with nvidia-smi
sampling the SM clock and board power, to show what the 1 kW power cap does to
launches that run longer than a burst.

`table4` sweeps lambda = a / L on the B200 shapes of the BLASST page's Table 4
(prefill: batch 148, 1 query / 1 KV head, 32K tokens, d 128, causal; decode:
batch 148, 32 query / 4 KV heads, 32K tokens, d 128) and reports, per a, the
skipped fraction and the speed-up over the same kernel with lambda = 0.

Used for Nsight Compute captures of a single kernel on a small case (a few
launches, a few hundred MB on the device) and for quick CUDA-event timings.
Prints one JSON line with the per-launch time and the algorithmic work.
"""
from __future__ import annotations

import argparse
import json

import torch

from . import inputs, ops

TILE = 2 * 128 * 128 * 128


def _time(fn, iters):
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record()
    for _ in range(iters):
        fn()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / iters


def table4(args):
    rows = []
    a_list = (0.0, 0.1, 1.0, 10.0, 100.0, 1000.0)
    # prefill: B148 H1 N32768 d128 causal (one query head per KV head)
    B, N = 148, 32768
    q, k, v = inputs.blasst_prefill_qkv(B, 1, 1, N, 128, "cuda", 4242)
    o = torch.empty_like(q)
    nq = N // 128
    base = None
    for a in a_list:
        lam = inputs.lambda_for(a, N)
        st = torch.zeros(B, 1, nq, nq, dtype=torch.uint8, device="cuda")
        ops.bsattn_fwd_prefill(q, k, v, 128, None, True, lam, o=o, tile_status=st, want_lse=False)
        torch.cuda.synchronize()
        vis, exe = int((st > 0).sum()), int((st == 2).sum())
        fn = lambda: ops.bsattn_fwd_prefill(q, k, v, 128, None, True, lam, o=o, want_lse=False)
        for _ in range(args.warmup):
            fn()
        ms = _time(fn, args.iters)
        base = ms if base is None else base
        rows.append({"kernel": "prefill", "a": a, "skipped": 1 - exe / vis, "ms": ms,
                     "speedup_vs_dense": base / ms, "tflops": TILE * (vis + exe) / ms / 1e9})
    del q, k, v, o
    torch.cuda.empty_cache()
    # decode: B148 Hq32/Hkv4 L32768 d128, 16 splits
    B, Hq, Hkv, L = 148, 32, 4, 32768
    q, k, v = inputs.blasst_decode_qkv(B, Hq, Hkv, L, 128, "cuda", 4243)
    T = L // 128
    ws = torch.empty(ops.bsattn_decode_workspace_size(B, Hq, 128, 16), dtype=torch.uint8,
                     device="cuda")
    o = torch.empty_like(q)
    base = None
    for a in a_list:
        lam = inputs.lambda_for(a, L)
        st = torch.zeros(B, Hkv, T, dtype=torch.uint8, device="cuda")
        ops.bsattn_fwd_decode(q, k, v, 128, 16, None, lam, o=o, workspace=ws, tile_status=st,
                              want_lse=False)
        torch.cuda.synchronize()
        vis, exe = int((st > 0).sum()), int((st == 2).sum())
        fn = lambda: ops.bsattn_fwd_decode(q, k, v, 128, 16, None, lam, o=o, want_lse=False,
                                           workspace=ws)
        for _ in range(args.warmup):
            fn()
        ms = _time(fn, args.iters)
        base = ms if base is None else base
        byt = 2 * B * Hq * 128 * 2 + 128 * 128 * 2 * (vis + exe)
        rows.append({"kernel": "decode", "a": a, "skipped": 1 - exe / vis, "ms": ms,
                     "speedup_vs_dense": base / ms, "gbs": byt / ms / 1e6})
    return rows


def varlen(args):
    """Causal BLASST prefill over a batch padded to N = 16384 with valid
    lengths 16384, 12288, 8192 and 4096 (32 query / 8 KV heads), against the
    same batch without lengths (every sequence full)."""
    B, H, Hkv, N = 4, 32, 8, 16384
    q, k, v = inputs.blasst_prefill_qkv(B, H, Hkv, N, 128, "cuda", 5150)
    lens = torch.tensor([16384, 12288, 8192, 4096], dtype=torch.int32, device="cuda")
    o = torch.empty_like(q)
    nq = N // 128
    rows = []
    for name, sl in (("padded_full", None), ("varlen", lens)):
        lam = inputs.lambda_for(args.a, N)
        st = torch.zeros(B, H, nq, nq, dtype=torch.uint8, device="cuda")
        ops.bsattn_fwd_prefill(q, k, v, 128, None, True, lam, o=o, tile_status=st, want_lse=False,
                               seq_lens=sl)
        torch.cuda.synchronize()
        vis, exe = int((st > 0).sum()), int((st == 2).sum())
        fn = lambda: ops.bsattn_fwd_prefill(q, k, v, 128, None, True, lam, o=o, want_lse=False,
                                            seq_lens=sl)
        for _ in range(args.warmup):
            fn()
        ms = _time(fn, args.iters)
        rows.append({"case": name, "a": args.a, "visited": vis, "executed": exe, "ms": ms,
                     "tflops": TILE * (vis + exe) / ms / 1e9})
    return rows


def backward(args):
    """Gradients of the causal BLASST prefill (B1, Hq heads, Hq/4 KV heads, N
    tokens, d 128) with the forward's executed tiles held fixed.  Work per
    executed tile: 5 GEMM tiles of 2*128*128*128 flops (S, dP, dV, dK, dQ);
    the kernels issue 7 (S and dP again for dQ)."""
    hkv = max(1, args.heads // 4)
    q, k, v = inputs.blasst_prefill_qkv(1, args.heads, hkv, args.n, 128, "cuda", 1237)
    lam = inputs.lambda_for(args.a, args.n)
    nq = args.n // 128
    st = torch.zeros(1, args.heads, nq, nq, dtype=torch.uint8, device="cuda")
    o, lse = ops.bsattn_fwd_prefill(q, k, v, 128, None, True, lam, tile_status=st)
    dout = torch.randn(q.shape, generator=torch.Generator(device="cuda").manual_seed(7),
                       device="cuda").to(torch.bfloat16)
    torch.cuda.synchronize()
    exe = int((st == 2).sum())
    fn = lambda: ops.bsattn_bwd_prefill(q, k, v, o, dout, lse, st, 128, None, True)  # noqa: E731
    for _ in range(args.warmup):
        fn()
    ms = _time(fn, args.iters)
    return {"heads": args.heads, "n": args.n, "a": args.a, "executed": exe, "ms": ms,
            "tflops": 5 * TILE * exe / ms / 1e9, "tflops_issued": 7 * TILE * exe / ms / 1e9}


def sustained(args):
    """Per-phase CUDA-event times with the SM clock and power sampled by
    nvidia-smi (every 50 ms) over each phase."""
    import datetime
    import subprocess
    import time
    pw = inputs.workload("blasst_prefill", device="cuda")
    dw = inputs.workload("blasst_decode", device="cuda")
    p_lam, d_lam = inputs.lambda_for(args.a, pw.N), inputs.lambda_for(args.a, dw.N)
    mask = torch.ones(1, pw.nq, pw.nk, dtype=torch.uint8, device="cuda")
    rp, ci, _, order = ops.bsattn_build_index(mask, 128, 128, True, with_order=True)
    o, lse = torch.empty_like(pw.q), torch.empty(pw.B, pw.Hq, pw.N, device="cuda")
    dout, dlse = torch.empty_like(dw.q), torch.empty(dw.B, dw.Hq, device="cuda")
    ws = torch.empty(ops.bsattn_decode_workspace_size(dw.B, dw.Hq, dw.d, dw.num_splits),
                     dtype=torch.uint8, device="cuda")

    def index():
        ops.bsattn_build_index(mask, 128, 128, True, with_order=True)

    def prefill():
        ops.bsattn_fwd_prefill(pw.q, pw.k, pw.v, 128, pw.scale, True, p_lam, rp, ci, 1, o=o,
                               lse=lse, row_order=order)

    def decode():
        ops.bsattn_fwd_decode(dw.q, dw.k, dw.v, 128, dw.num_splits, dw.scale, d_lam, o=dout,
                              lse=dlse, workspace=ws)

    def idle():
        torch.cuda._sleep(20_000_000)   # about 10 ms

    prefill(), decode()
    torch.cuda.synchronize()
    smi = subprocess.Popen(["nvidia-smi", "--query-gpu=timestamp,clocks.sm,power.draw,"
                            "clocks_event_reasons.sw_power_cap", "--format=csv,noheader",
                            "-lms", "50"], stdout=subprocess.PIPE, text=True)
    phases = [("prefill alone", [prefill], 200), ("step", [index, prefill, decode], 100),
              ("step + 10 ms idle", [index, prefill, decode, idle], 40),
              ("decode alone", [decode], 200)]
    res = []
    stream = torch.cuda.current_stream()
    for name, fns, n in phases:
        idle()
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(fns) + 1)]
              for _ in range(n)]
        t0 = time.time()
        for i in range(n):
            ev[i][0].record(stream)
            for j, f in enumerate(fns):
                f()
                ev[i][j + 1].record(stream)
        torch.cuda.synchronize()
        t1 = time.time()
        ms = [[ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(n)] for j in range(len(fns))]
        res.append({"phase": name, "t": (t0, t1),
                    "first5_ms": [round(sum(m[:5]) / 5, 3) for m in ms],
                    "rest_ms": [round(sum(m[n // 4:]) / (n - n // 4), 3) for m in ms]})
    time.sleep(0.2)
    smi.terminate()
    txt, _ = smi.communicate()
    samples = []
    for line in txt.strip().splitlines():
        f = [x.strip() for x in line.split(",")]
        try:
            ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            samples.append((ts, float(f[1].split()[0]), float(f[2].split()[0]),
                            f[3].lower().startswith("active")))
        except (ValueError, IndexError):
            continue
    for r in res:
        t0, t1 = r.pop("t")
        sel = [x for x in samples if t0 <= x[0] <= t1]
        if sel:
            mhz, watts = sorted(x[1] for x in sel), sorted(x[2] for x in sel)
            r.update(sm_mhz_median=mhz[len(mhz) // 2], power_w_median=watts[len(watts) // 2],
                     capped_samples=sum(x[3] for x in sel), samples=len(sel))
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("what", choices=("prefill", "decode", "videodit", "mmdit", "table4",
                                     "varlen", "backward", "sustained"))
    ap.add_argument("--heads", type=int, default=8, help="query heads (prefill/videodit/mmdit)")
    ap.add_argument("--n", type=int, default=32768, help="sequence length (prefill)")
    ap.add_argument("--batch", type=int, default=64, help="batch (decode)")
    ap.add_argument("--l", type=int, default=131072, help="KV length (decode)")
    ap.add_argument("--hkv", type=int, default=8, help="KV heads (decode; 32 query heads)")
    ap.add_argument("--splits", type=int, default=16, help="KV splits (decode)")
    ap.add_argument("--block", type=int, default=128, help="key tile (decode): 64 or 128")
    ap.add_argument("--a", type=float, default=10.0)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--no-order", action="store_true", help="static masks: no longest-first order")
    ap.add_argument("--dense-mask", action="store_true",
                    help="videodit/mmdit: an all-ones mask of the same shape (same kernel)")
    ap.add_argument("--diag-mask", action="store_true",
                    help="videodit/mmdit: only the diagonal block of every row")
    ap.add_argument("--reverse", action="store_true", help="prefill: descending visit order")
    ap.add_argument("--skip-v", action="store_true", help="prefill: load V only for kept tiles")
    ap.add_argument("--sink-seed", action="store_true", help="decode: sink-seeded splits")
    args = ap.parse_args()
    torch.cuda.set_device(0)
    out = {"what": args.what}
    if args.what == "prefill":
        hkv = max(1, args.heads // 4)
        q, k, v = inputs.blasst_prefill_qkv(1, args.heads, hkv, args.n, 128, "cuda", 1237)
        lam = inputs.lambda_for(args.a, args.n)
        nq = args.n // 128
        st = torch.zeros(1, args.heads, nq, nq, dtype=torch.uint8, device="cuda")
        opt = dict(reverse=args.reverse, skip_v=args.skip_v)
        if args.diag_mask:   # one key tile per query tile: the per-work-item cost
            m = torch.eye(nq, dtype=torch.uint8)[None].cuda()
            rp, ci, _ = ops.bsattn_build_index(m, 128, 128, True)
            opt.update(row_ptr=rp, col_idx=ci, mask_heads=1)
        o, _ = ops.bsattn_fwd_prefill(q, k, v, 128, None, True, lam, tile_status=st, **opt)
        torch.cuda.synchronize()
        vis, exe = int((st > 0).sum()), int((st == 2).sum())
        fn = lambda: ops.bsattn_fwd_prefill(q, k, v, 128, None, True, lam, o=o, want_lse=False,
                                            **opt)
        for _ in range(args.warmup):
            fn()
        ms = _time(fn, args.iters)
        out.update(heads=args.heads, n=args.n, a=args.a, reverse=args.reverse,
                   skip_v=args.skip_v, visited=vis, executed=exe, ms=ms,
                   tflops=TILE * (vis + exe) / ms / 1e9)
    elif args.what in ("videodit", "mmdit"):
        w = inputs.workload(args.what, device="cuda", generate=False)
        q, k, v = inputs.normal_qkv(1, args.heads, args.heads, w.N, w.d, "cuda", 1236)
        if args.dense_mask:
            m = torch.ones_like(w.mask).cuda()
        elif args.diag_mask:   # one key tile per query tile: the per-work-item cost
            m = torch.eye(w.nq, dtype=torch.uint8)[None].cuda()
        else:
            m = w.mask.cuda()
        rp, ci, nnz, order = ops.bsattn_build_index(m, w.block, w.block, False, with_order=True)
        if args.no_order:
            order = None
        fn = lambda: ops.bsattn_fwd_prefill(q, k, v, w.block, w.scale, False, 0.0, rp, ci, 1,
                                            want_lse=False, row_order=order)
        for _ in range(args.warmup):
            fn()
        ms = _time(fn, args.iters)
        tiles = int(nnz.sum()) * args.heads
        flops = 4 * w.block * w.block * w.d * tiles
        out.update(heads=args.heads, n=w.N, d=w.d, tiles=tiles, dense_mask=args.dense_mask, ms=ms,
                   tflops=flops / ms / 1e9)
    elif args.what == "table4":
        out["rows"] = table4(args)
    elif args.what == "varlen":
        out["rows"] = varlen(args)
    elif args.what == "backward":
        out.update(backward(args))
    elif args.what == "sustained":
        out["phases"] = sustained(args)
    else:
        B, Hq, Hkv, L, d = args.batch, 32, args.hkv, args.l, 128
        ns = args.splits
        q, k, v = inputs.blasst_decode_qkv(B, Hq, Hkv, L, d, "cuda", 1238)
        lam = inputs.lambda_for(args.a, L)
        blk = args.block
        T = -(-L // blk)
        st = torch.zeros(B, Hkv, T, dtype=torch.uint8, device="cuda")
        ws = torch.empty(ops.bsattn_decode_workspace_size(B, Hq, d, ns), dtype=torch.uint8,
                         device="cuda")
        o, _ = ops.bsattn_fwd_decode(q, k, v, blk, ns, None, lam, workspace=ws, tile_status=st,
                                     sink_seed=args.sink_seed)
        torch.cuda.synchronize()
        vis, exe = int((st > 0).sum()), int((st == 2).sum())
        fn = lambda: ops.bsattn_fwd_decode(q, k, v, blk, ns, None, lam, o=o, want_lse=False,
                                           workspace=ws, sink_seed=args.sink_seed)
        for _ in range(args.warmup):
            fn()
        ms = _time(fn, args.iters)
        byt = 2 * B * Hq * d * 2 + blk * d * 2 * (vis + exe)
        out.update(batch=B, l=L, hkv=Hkv, splits=ns, block=blk, sink_seed=args.sink_seed, a=args.a,
                   visited=vis, executed=exe, ms=ms, gbs=byt / ms / 1e6)
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
