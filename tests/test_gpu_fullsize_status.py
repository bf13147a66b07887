"""Whole-launch executed-tile sets at full size: every visited tile of the
full BLASST prefill (B1, 32 query / 8 KV heads, 32768 tokens, causal) at
a = 1, 10 and 100, every tile of the full BLASST decode (64 sequences of
131072 keys, 16 splits) at the same a, and every tile of the full
multimodal-DiT and Video-DiT masks -- against the oracle's first pass
(oracle/tile_margins.py, pinned to the C oracle on the CPU).

Decisions must match exactly except for tiles whose skip margin lies within
1e-3 of zero (BLASST page, section 3.1.1: the decision compares a tile's row
maxima with the running maxima; rounding may flip a near-tie).  The number of
such near-ties is printed.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_bsattn_b200 import inputs
from oracle import tile_margins
from tests.parity import MARGIN_TIE, compare_status

pytestmark = pytest.mark.gpu


def _ops():
    from block_sparse_attention_bsattn_b200 import ops
    return ops


def _report(what, st, ref_status, ref_margin):
    differ = compare_status(st, ref_status, ref_margin, what)
    near = int((np.abs(ref_margin) < MARGIN_TIE).sum())
    vis = int((ref_status > 0).sum())
    ex = int((ref_status == 2).sum())
    print(f"{what}: {vis} visited, {ex} executed, {near} near-ties, {differ} differ")


@pytest.fixture(scope="module")
def blasst_prefill_full():
    w = inputs.workload("blasst_prefill", device="cuda")
    D = tile_margins.prefill_margins(w.q, w.k, w.block, w.scale, w.causal)
    return w, D


@pytest.mark.parametrize("a", [1.0, 10.0, 100.0])
def test_blasst_prefill_full_size_whole_tile_set(blasst_prefill_full, a):
    ops = _ops()
    w, D = blasst_prefill_full
    lam = inputs.lambda_for(a, w.N)
    st = torch.zeros(w.B, w.Hq, w.nq, w.nk, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.bsattn_fwd_prefill(w.q, w.k, w.v, w.block, w.scale, True, lam, tile_status=st,
                           status=status, want_lse=False)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref_st, ref_mg = tile_margins.status_from_margins(D, lam)
    _report(f"blasst prefill a={a}", st.cpu().numpy(), ref_st, ref_mg)


@pytest.fixture(scope="module")
def blasst_decode_full():
    w = inputs.workload("blasst_decode", device="cuda")
    yield w
    del w
    torch.cuda.empty_cache()


# the workload's 16 splits at a = 1, 10, 100, and the benchmark's decode
# operating point (4 splits at a = 160)
@pytest.mark.parametrize("a,splits", [(1.0, 16), (10.0, 16), (100.0, 16),
                                      (inputs.DECODE_OP_A, inputs.DECODE_OP_SPLITS)])
def test_blasst_decode_full_size_whole_tile_set(blasst_decode_full, a, splits):
    ops = _ops()
    w = blasst_decode_full
    lam = inputs.lambda_for(a, w.N)
    T = -(-w.N // w.block)
    st = torch.zeros(w.B, w.Hkv, T, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.bsattn_fwd_decode(w.q, w.k, w.v, w.block, splits, w.scale, lam, tile_status=st,
                          status=status, want_lse=False)
    torch.cuda.synchronize()
    assert status.item() == 0
    D = tile_margins.decode_margins(w.q, w.k, w.block, w.scale, splits)
    ref_st, ref_mg = tile_margins.status_from_margins(D, lam)
    _report(f"blasst decode a={a} splits={splits}", st.cpu().numpy().reshape(w.B * w.Hkv, T),
            ref_st, ref_mg)


@pytest.mark.parametrize("name", ["mmdit", "videodit"])
def test_static_mask_full_size_whole_tile_set(name):
    """lambda = 0 with a static block mask: the executed set of every query
    head is the mask itself (every kept block visited and executed, no
    other), bit for bit."""
    ops = _ops()
    w = inputs.workload(name, device="cuda")
    m = w.mask.cuda()
    rp, ci, _, order = ops.bsattn_build_index(m, w.block, w.block, False, with_order=True)
    st = torch.zeros(w.B, w.Hq, w.nq, w.nk, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.bsattn_fwd_prefill(w.q, w.k, w.v, w.block, w.scale, False, 0.0, rp, ci, 1, tile_status=st,
                           status=status, row_order=order, want_lse=False)
    torch.cuda.synchronize()
    assert status.item() == 0
    expect = (w.mask.numpy()[0].astype(np.uint8) * 2)[None, None]
    got = st.cpu().numpy()
    assert (got == expect).all(), f"{name}: {int((got != expect).sum())} tiles differ"
    print(f"{name}: {int((got == 2).sum())} executed tiles over {w.Hq} heads, all as the mask")
