"""Sweep the attention-sink strength of the BLASST prefill input recipe with the
CPU oracle and report the skipped fraction of visited tiles at a = 10
(lambda = a / N).  Used once to fix ``inputs.SINK_BETA`` so that the
synthetic workload sits near the 74.7% prefill sparsity the BLASST page
reports (section A1); the chosen value and this script's output are kept in
tests/golden/sink_beta.txt.

    python tests/golden/calibrate_sink_beta.py [--betas 0,1,2,3] [--items 16]
"""
import argparse
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from block_sparse_attention_bsattn_b200 import inputs  # noqa: E402


def skipped_fraction(beta, n_items, a=10.0, seed=1237, hq=8, hkv=2):
    N, d, block = 32768, 128, 128
    q, k, v = inputs.blasst_prefill_qkv(1, hq, hkv, N, d, "cpu", seed, sink_beta=beta)
    nq = N // block
    rng = np.random.default_rng(0)
    items = sorted({(0, int(rng.integers(hq)), int(rng.integers(nq))) for _ in range(n_items)})
    r = oracle.prefill(q, k, v, block, 1 / np.sqrt(d), True, inputs.lambda_for(a, N), items=items)
    st = r["status"]
    return 1 - (st == 2).sum() / (st > 0).sum()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--betas", default="0,1,2,3,4")
    ap.add_argument("--items", type=int, default=16)
    a = ap.parse_args()
    for b in [float(x) for x in a.betas.split(",")]:
        print(f"beta={b:g} skipped_fraction(a=10)={skipped_fraction(b, a.items):.3f}", flush=True)


if __name__ == "__main__":
    main()
