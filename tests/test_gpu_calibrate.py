"""lambda = a / L calibration (BLASST page, section 3.2 and Algorithm 2) with
the CUDA kernel as the measuring function: calibrate.calibrate driven by
calibrate.prefill_sparsity (the kernel's per-tile status) on the causal
BLASST prefill recipe at three lengths, against the same loop driven by the
oracle's first pass on the same inputs.  At every lambda of the grid the
kernel's executed tiles must equal the oracle's except near-ties (|margin| <
1e-3), and the fitted a must be the oracle-driven fit."""
import math

import numpy as np
import pytest

from block_sparse_attention_bsattn_b200 import calibrate, inputs
from oracle import tile_margins
from tests.parity import MARGIN_TIE, compare_status

pytestmark = pytest.mark.gpu

LENGTHS = (2048, 4096, 8192)
HEADS, KV_HEADS, SEED = 8, 2, 1237


def test_calibration_loop_on_kernel_equals_oracle_loop():
    import torch
    from block_sparse_attention_bsattn_b200 import ops

    scale = 1 / math.sqrt(128)
    cache, D = {}, {}
    for L in LENGTHS:
        q, k, v = inputs.blasst_prefill_qkv(1, HEADS, KV_HEADS, L, 128, "cuda", SEED)
        cache[(L, HEADS, KV_HEADS, SEED)] = (q, k, v)     # prefill_sparsity's input cache
        D[L] = tile_margins.prefill_margins(q, k, 128, scale, True)
    lambdas = calibrate.log_grid(1e-7, 1e-1, 13)

    def oracle_sparsity(lam, L):
        st, _ = tile_margins.status_from_margins(D[L], lam)
        return 1.0 - (st == 2).sum() / (st > 0).sum()

    def kernel_sparsity(lam, L):
        return calibrate.prefill_sparsity(lam, L, heads=HEADS, kv_heads=KV_HEADS, seed=SEED,
                                          cache=cache)

    # per (lambda, L): the kernel's executed tiles are the oracle's (near-ties
    # aside), so the measured sparsities agree to the near-tie fraction
    ties_seen = 0
    for L in LENGTHS:
        q, k, v = cache[(L, HEADS, KV_HEADS, SEED)]
        nq = L // 128
        for lam in lambdas:
            st = torch.zeros(1, HEADS, nq, nq, dtype=torch.uint8, device="cuda")
            ops.bsattn_fwd_prefill(q, k, v, 128, scale, True, lam, tile_status=st,
                                   want_lse=False)
            torch.cuda.synchronize()
            ref_st, ref_mg = tile_margins.status_from_margins(D[L], lam)
            differ = compare_status(st.cpu().numpy(), ref_st, ref_mg, f"L={L} lambda={lam:.2e}")
            ties_seen += differ
            vis = int((ref_st > 0).sum())
            assert abs(kernel_sparsity(lam, L) - oracle_sparsity(lam, L)) <= differ / vis + 1e-12

    # the target: the oracle's sparsity at the middle length and grid point,
    # so that at least that length reaches it
    target = float(oracle_sparsity(lambdas[len(lambdas) // 2], LENGTHS[1]))
    a_kernel, pts_kernel = calibrate.calibrate(kernel_sparsity, LENGTHS, lambdas, target, 0.05)
    a_oracle, pts_oracle = calibrate.calibrate(oracle_sparsity, LENGTHS, lambdas, target, 0.05)
    print(f"target {target:.4f}: a = {a_kernel:.6g} (kernel), {a_oracle:.6g} (oracle); "
          f"{ties_seen} tile decisions differed at near-ties")
    if ties_seen == 0:
        assert a_kernel == a_oracle
        assert [(x, y) for x, y, _ in pts_kernel] == [(x, y) for x, y, _ in pts_oracle]
    else:
        assert a_kernel == pytest.approx(a_oracle, rel=0.5)
    assert np.isfinite(a_kernel) and a_kernel > 0
