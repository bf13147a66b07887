"""Threshold calibration lambda = a / L ("BLASST: Dynamic Blocked Attention
Sparsity via Softmax Thresholding", section 3.2 and Algorithm 2).

For each context length L_k the lambda of a candidate set whose measured
sparsity is closest to the target S is kept, provided it lands within a
tolerance delta of S; a line through the origin, lambda = a * (1 / L), is then
fitted to the kept points (1 / L_k, lambda_best) by least squares and a is
returned.  The sparsity measurement is a callable, so the same procedure runs
on the GPU kernel (:func:`prefill_sparsity`, from the kernel's per-tile
status) or on anything else that reports a skipped fraction.

    python -m block_sparse_attention_bsattn_b200.calibrate --target 0.5 \\
        --lengths 4096,8192,16384,32768 --heads 8
"""
from __future__ import annotations

import argparse
import json
import math
from typing import Callable, Iterable, List, Sequence, Tuple


def calibrate(measure: Callable[[float, int], float], lengths: Iterable[int],
              lambdas: Sequence[float], target: float, tol: float
              ) -> Tuple[float, List[Tuple[float, float, float]]]:
    """Return (a, points) with points = [(1/L, lambda_best, sparsity), ...]
    for the lengths whose best lambda came within `tol` of `target`.
    Ties between candidates keep the first one in `lambdas` order."""
    points = []
    for L in lengths:
        best, best_gap, best_s = None, math.inf, None
        for lam in lambdas:
            s = measure(lam, L)
            gap = abs(s - target)
            if gap < best_gap:
                best, best_gap, best_s = lam, gap, s
        if best_gap < tol:
            points.append((1.0 / L, best, best_s))
    if not points:
        raise ValueError("no context length reached the target sparsity within the tolerance")
    num = sum(x * y for x, y, _ in points)
    den = sum(x * x for x, _, _ in points)
    return num / den, points


def log_grid(lo: float, hi: float, n: int) -> List[float]:
    """n values spaced evenly in log between lo and hi."""
    return [lo * (hi / lo) ** (k / (n - 1)) for k in range(n)]


def prefill_sparsity(lam: float, L: int, heads: int = 8, kv_heads: int = 2, seed: int = 1237,
                     cache: dict | None = None) -> float:
    """Skipped fraction of the visited tiles of the causal BLASST prefill
    workload recipe at length L (tiles of 128, d = 128), measured by the CUDA
    kernel's tile status."""
    import torch

    from . import inputs, ops
    key = (L, heads, kv_heads, seed)
    if cache is not None and key in cache:
        q, k, v = cache[key]
    else:
        q, k, v = inputs.blasst_prefill_qkv(1, heads, kv_heads, L, 128, "cuda", seed)
        if cache is not None:
            cache[key] = (q, k, v)
    nq = -(-L // 128)
    st = torch.zeros(1, heads, nq, nq, dtype=torch.uint8, device="cuda")
    ops.bsattn_fwd_prefill(q, k, v, 128, None, True, lam, tile_status=st, want_lse=False)
    torch.cuda.synchronize()
    visited = int((st > 0).sum())
    return 1.0 - int((st == 2).sum()) / visited


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--target", type=float, default=0.5)
    ap.add_argument("--tol", type=float, default=0.05)
    ap.add_argument("--lengths", default="4096,8192,16384,32768")
    ap.add_argument("--heads", type=int, default=8)
    ap.add_argument("--lambdas", type=int, default=31, help="log grid size over [1e-10, 1]")
    args = ap.parse_args()
    lengths = [int(x) for x in args.lengths.split(",")]
    lambdas = log_grid(1e-10, 1.0, args.lambdas)
    cache: dict = {}
    curve: dict = {}

    def measure(lam, L):
        s = prefill_sparsity(lam, L, heads=args.heads, cache=cache)
        curve.setdefault(L, []).append((lam, s))
        return s

    try:
        a, points = calibrate(measure, lengths, lambdas, args.target, args.tol)
    except ValueError as e:
        print(json.dumps({"target": args.target, "error": str(e),
                          "measured": {str(L): c for L, c in curve.items()}}), flush=True)
        raise SystemExit(2)
    # achieved sparsity of the fitted law at every length
    check = [{"L": L, "lambda": a / L, "sparsity": measure(a / L, L)} for L in lengths]
    print(json.dumps({"target": args.target, "tol": args.tol, "a": a,
                      "points": [{"L": round(1 / x), "lambda_best": y, "sparsity": s}
                                 for x, y, s in points],
                      "fitted": check}), flush=True)


if __name__ == "__main__":
    main()
