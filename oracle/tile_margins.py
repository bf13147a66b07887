"""Pass 1 of the BLASST visit on its own: the skip margin of every visited
tile, for whole workloads -- TEST INFRASTRUCTURE, under the same rules as the
rest of ``oracle/`` (only tests, the smoke check and the benchmark's CPU
baseline may use it; nothing here is shared with the CUDA library).

"BLASST: Dynamic Blocked Attention Sparsity via Softmax Thresholding",
Algorithm 1 and section 3.1.1: a query tile visits its key tiles in order;
for each, every row's tile maximum of the scaled scores is compared with the
row's running maximum over the tiles visited before it, and the tile is
skipped when every row's difference lies below ln(lambda).  The difference
kept here is the largest one over the valid rows,

    D_j = max_r (max_c S_rc - m_prev_r),   S = scale * Q K^T,

with (-inf) - (-inf) counted as +inf (the test cannot pass).  Because a
skipped tile never raises the running maximum when lambda <= 1, m_prev is
the maximum over all earlier visited tiles whatever was skipped, so one D per
tile gives the decision for every lambda: skipped iff lambda > 0 and
D_j < ln(lambda); the margin the full oracle reports is D_j - ln(lambda).

This is the same first pass as ``oracle_prefill`` / ``oracle_decode`` in
``bsattn_oracle.c`` (whose second pass, the exact softmax over the executed
tiles, is not needed for the tile sets), with the score products taken from
an fp64 matrix product -- a library primitive -- so that whole workloads of
a few TFLOP finish in about a minute on the host cores.  Its agreement with
the C oracle is pinned on the CPU (tests/test_oracle_margins.py).
"""
from __future__ import annotations

import math

import numpy as np
import torch


def _f64(x: torch.Tensor) -> torch.Tensor:
    """bf16 (or any float) tensor -> fp64 on the CPU; exact for bf16."""
    return x.detach().to("cpu").to(torch.float64)


def prefill_margins(q: torch.Tensor, k: torch.Tensor, block: int, scale: float, causal: bool,
                    heads=None, rows_per_step: int = 1024) -> np.ndarray:
    """D for every (query head, query tile, key tile) of a prefill whose
    visit list is every key tile (causal: the key tiles up to the diagonal),
    in ascending order, sequences of full length.

    q [B,Hq,N,d], k [B,Hkv,N,d].  heads: None (all) or a list of query-head
    indices.  Returns float64 [B, len(heads), nq, nk]: D of each visited tile,
    NaN where the tile is not visited."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    nq = -(-N // block)
    heads = list(range(Hq)) if heads is None else list(heads)
    out = np.full((B, len(heads), nq, nq), np.nan)
    rows_per_step = max(block, (rows_per_step // block) * block)
    for b in range(B):
        kcache = {}
        for hi, h in enumerate(heads):
            kvh = h // g
            if kvh not in kcache:
                kcache = {kvh: _f64(k[b, kvh])}
            kf = kcache[kvh]
            qf = _f64(q[b, h])
            for r0 in range(0, N, rows_per_step):
                r1 = min(N, r0 + rows_per_step)
                # keys any of these rows may see
                kend = min(N, ((r1 - 1) // block + 1) * block) if causal else N
                s = (qf[r0:r1] @ kf[:kend].T) * scale               # [rows, kend]
                if causal:
                    qpos = torch.arange(r0, r1).unsqueeze(1)
                    key = torch.arange(kend).unsqueeze(0)
                    s = s.masked_fill(key > qpos, -math.inf)
                nt = -(-kend // block)
                pad = nt * block - kend
                if pad:
                    s = torch.nn.functional.pad(s, (0, pad), value=-math.inf)
                tmax = s.view(r1 - r0, nt, block).amax(dim=2)       # [rows, nt]
                # running max before each tile, in visit (ascending) order
                prev = torch.cummax(tmax, dim=1).values
                mprev = torch.cat([torch.full((r1 - r0, 1), -math.inf, dtype=torch.float64),
                                   prev[:, :-1]], dim=1)
                dr = tmax - mprev
                dr = torch.where(torch.isnan(dr), torch.full_like(dr, math.inf), dr)
                for i in range(r0 // block, (r1 - 1) // block + 1):
                    lo, hi_ = max(i * block, r0) - r0, min((i + 1) * block, r1) - r0
                    nvis = min(i + 1, nt) if causal else nt
                    out[b, hi, i, :nvis] = dr[lo:hi_, :nvis].amax(dim=0).numpy()
    return out


def decode_margins(q: torch.Tensor, k: torch.Tensor, block: int, scale: float,
                   num_splits: int, pairs=None, sink_seed: bool = False) -> np.ndarray:
    """D for every key tile of a split-KV decode: the query tile is the GQA
    group of one token (all g rows valid), the KV tiles are cut into
    num_splits contiguous chunks of ceil(T / num_splits) tiles, and the
    running max starts from -inf at each chunk start -- or, with sink_seed,
    every chunk after the first starts from the row maxima of key tile 0 (the
    tile of the attention sink), scored but not visited.

    q [B,Hq,d], k [B,Hkv,L,d].  pairs: None (every (b, kv head)) or a list
    of (b, kv head).  Returns float64 [len(pairs), T]."""
    B, Hq, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    g = Hq // Hkv
    T = -(-L // block)
    chunk = -(-T // num_splits)
    pairs = [(b, h) for b in range(B) for h in range(Hkv)] if pairs is None else list(pairs)
    out = np.empty((len(pairs), T))
    for p, (b, kvh) in enumerate(pairs):
        kf = _f64(k[b, kvh])                                      # [L, d]
        qf = _f64(q[b, kvh * g:(kvh + 1) * g])                    # [g, d]
        s = (qf @ kf.T) * scale                                   # [g, L]
        pad = T * block - L
        if pad:
            s = torch.nn.functional.pad(s, (0, pad), value=-math.inf)
        tmax = s.view(g, T, block).amax(dim=2)                    # [g, T]
        for c0 in range(0, T, chunk):
            c1 = min(T, c0 + chunk)
            tm = tmax[:, c0:c1]
            prev = torch.cummax(tm, dim=1).values
            start = torch.full((g, 1), -math.inf, dtype=torch.float64)
            if sink_seed and c0 > 0:
                start = tmax[:, :1].clone()
            mprev = torch.cat([start, torch.maximum(prev[:, :-1], start)], dim=1)
            dr = tm - mprev
            dr = torch.where(torch.isnan(dr), torch.full_like(dr, math.inf), dr)
            out[p, c0:c1] = dr.amax(dim=0).numpy()
    return out


def status_from_margins(D: np.ndarray, lam: float):
    """(status, margin) for one lambda from D: status 0 not visited (D NaN),
    1 skipped (lambda > 0 and D < ln lambda), 2 executed; margin D - ln
    lambda, +inf when lambda = 0 (the test cannot pass)."""
    visited = ~np.isnan(D)
    status = np.zeros(D.shape, np.uint8)
    if lam > 0:
        ln = math.log(lam)
        with np.errstate(invalid="ignore"):
            skip = visited & (D < ln)
        margin = np.where(visited, D - ln, np.nan)
    else:
        skip = np.zeros(D.shape, bool)
        margin = np.where(visited, np.inf, np.nan)
    status[visited] = 2
    status[skip] = 1
    return status, margin
