"""Pins of oracle/tile_margins.py (the first pass of the BLASST visit alone,
used to check whole-launch executed-tile sets at full size) against the C
oracle's own first pass, on the shrunk workloads and on shapes with ragged
tails, GQA and both causal settings: the same status for every lambda, the
same margins."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_bsattn_b200 import inputs
from oracle import tile_margins


def _same_margins(got, ref, visited):
    both_inf = np.isposinf(got) & np.isposinf(ref)
    both_ninf = np.isneginf(got) & np.isneginf(ref)
    fin = visited & ~both_inf & ~both_ninf
    assert np.isfinite(got[fin]).all() and np.isfinite(ref[fin]).all()
    assert np.abs(got[fin] - ref[fin]).max(initial=0.0) < 1e-9


@pytest.mark.parametrize("a", [0.0, 1.0, 10.0, 100.0])
def test_prefill_margins_equal_oracle_on_shrunk_blasst_prefill(a):
    w = inputs.workload("blasst_prefill", shrink=True)
    lam = inputs.lambda_for(a, w.N)
    D = tile_margins.prefill_margins(w.q, w.k, w.block, w.scale, w.causal)
    st, mg = tile_margins.status_from_margins(D, lam)
    ref = oracle.prefill(w.q, w.k, w.v, w.block, w.scale, w.causal, lam)
    assert (st == ref["status"]).all()
    _same_margins(mg, ref["margin"], ref["status"] > 0)
    if a >= 10:
        assert (st == 1).sum() > 0 and (st == 2).sum() > 0


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [3 * 128, 4 * 128 - 37])
def test_prefill_margins_ragged_gqa(causal, N):
    """GQA 3, non-multiple lengths (the last query tile and key tile are
    partial), rows processed in steps that do not align with the tiles."""
    q, k, v = inputs.blasst_prefill_qkv(2, 3, 1, N, 64, "cpu", 55 + N)
    lam = 2e-2
    D = tile_margins.prefill_margins(q, k, 128, 0.125, causal, rows_per_step=256)
    st, mg = tile_margins.status_from_margins(D, lam)
    ref = oracle.prefill(q, k, v, 128, 0.125, causal, lam)
    assert (st == ref["status"]).all()
    _same_margins(mg, ref["margin"], ref["status"] > 0)
    # a subset of the heads gives those heads' rows
    Dh = tile_margins.prefill_margins(q, k, 128, 0.125, causal, heads=[2])
    np.testing.assert_array_equal(np.isnan(Dh[:, 0]), np.isnan(D[:, 2]))
    fin = ~np.isnan(Dh[:, 0])
    assert np.allclose(Dh[:, 0][fin], D[:, 2][fin], rtol=0, atol=1e-12)


@pytest.mark.parametrize("a", [1.0, 10.0, 100.0])
def test_decode_margins_equal_oracle_on_shrunk_blasst_decode(a):
    w = inputs.workload("blasst_decode", shrink=True)
    lam = inputs.lambda_for(a, w.N)
    D = tile_margins.decode_margins(w.q, w.k, w.block, w.scale, w.num_splits)
    st, mg = tile_margins.status_from_margins(D, lam)
    g = w.Hq // w.Hkv
    pairs = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    qs, ks, vs = oracle.decode_problems(w.q, w.k, w.v, pairs)
    ref = oracle.decode(qs, ks, vs, w.block, w.scale, lam, w.num_splits)
    assert g == qs.shape[1]
    assert (st == ref["status"]).all()
    _same_margins(mg, ref["margin"], ref["status"] > 0)


@pytest.mark.parametrize("a", [0.01, 1.0, 10.0])
def test_decode_margins_sink_seed_equal_oracle(a):
    """Sink-seeded splits: every split after the first starts its running max
    from key tile 0's row maxima."""
    w = inputs.workload("blasst_decode", shrink=True)
    lam = inputs.lambda_for(a, w.N)
    D = tile_margins.decode_margins(w.q, w.k, w.block, w.scale, w.num_splits, sink_seed=True)
    st, mg = tile_margins.status_from_margins(D, lam)
    pairs = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    qs, ks, vs = oracle.decode_problems(w.q, w.k, w.v, pairs)
    ref = oracle.decode(qs, ks, vs, w.block, w.scale, lam, w.num_splits, sink_seed=True)
    assert (st == ref["status"]).all()
    _same_margins(mg, ref["margin"], ref["status"] > 0)
    plain, _ = tile_margins.status_from_margins(
        tile_margins.decode_margins(w.q, w.k, w.block, w.scale, w.num_splits), lam)
    assert (st == 1).sum() >= (plain == 1).sum()


def test_status_from_margins_closed_form():
    """D = NaN: not visited; lambda = 0: every visited tile executed with an
    infinite margin; otherwise skipped exactly when D < ln lambda, including
    D = -inf (every row fully masked) and never for D = +inf."""
    D = np.array([np.nan, math.inf, -math.inf, -3.0, -1.0, 0.0])
    st, mg = tile_margins.status_from_margins(D, 0.0)
    assert st.tolist() == [0, 2, 2, 2, 2, 2]
    assert np.isposinf(mg[1:]).all() and np.isnan(mg[0])
    st, mg = tile_margins.status_from_margins(D, math.exp(-2.0))
    assert st.tolist() == [0, 2, 1, 1, 2, 2]
    assert abs(mg[3] - (-1.0)) < 1e-12
