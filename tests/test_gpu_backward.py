"""Backward parity: bsattn_bwd_prefill against the oracle's prefill_bwd.

The GPU forward runs first (its tile status and LSE are the backward's
inputs); the oracle's backward takes the same tile status, so both sides hold
the same executed set, and its forward decisions are checked against the
oracle's own by the forward tests.  Gradients are compared relative to the
largest reference magnitude of each tensor: the GPU path rounds P and dS to
bf16 for the tensor cores and accumulates in fp32."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_bsattn_b200 import inputs

pytestmark = pytest.mark.gpu


def _ops():
    from block_sparse_attention_bsattn_b200 import ops
    return ops


def _cmp(got, ref, what, tol_max=3e-2, tol_mean=3e-3):
    g = got.float().cpu().numpy().astype(np.float64)
    scale = max(np.abs(ref).max(), 1e-6)
    err = np.abs(g - ref)
    assert err.max() <= tol_max * scale, f"{what}: max err {err.max():.3e} vs {scale:.3e}"
    assert err.mean() <= tol_mean * scale, f"{what}: mean err {err.mean():.3e} vs {scale:.3e}"


def _run(q, k, v, causal, lam, mask=None, seq_lens=None, seed=0):
    ops = _ops()
    B, Hq, N, d = q.shape
    block = 128
    nq = -(-N // block)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    rp = ci = None
    mh = 1
    if mask is not None:
        rp, ci, _ = ops.bsattn_build_index(torch.as_tensor(mask).cuda(), block, block, causal)
        mh = mask.shape[0]
    st = torch.zeros(B, Hq, nq, nq, dtype=torch.uint8, device="cuda")
    sl = None if seq_lens is None else torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    o, lse = ops.bsattn_fwd_prefill(qd, kd, vd, block, 1 / math.sqrt(d), causal, lam, rp, ci, mh,
                                    tile_status=st, seq_lens=sl)
    g = torch.Generator().manual_seed(seed)
    dout = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dk, dv = ops.bsattn_bwd_prefill(qd, kd, vd, o, dout.cuda(), lse, st, block,
                                        1 / math.sqrt(d), causal, seq_lens=sl, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = oracle.prefill_bwd(q, k, v, dout, block, 1 / math.sqrt(d), causal, st.cpu().numpy(),
                             seq_lens=seq_lens)
    return (dq, dk, dv), ref, st


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_dense(d, causal):
    q, k, v = inputs.normal_qkv(1, 4, 2, 5 * 128 + 37, d, "cpu", 31)
    (dq, dk, dv), ref, _ = _run(q, k, v, causal, 0.0)
    _cmp(dq, ref["dq"], "dq")
    _cmp(dk, ref["dk"], "dk")
    _cmp(dv, ref["dv"], "dv")


@pytest.mark.parametrize("a", [1.0, 10.0, 100.0])
def test_bwd_blasst(a):
    """The BLASST recipe with a weaker sink (2 instead of 3.4): 27-40% of the
    visited tiles skipped and gradients of ordinary size."""
    B, Hq, Hkv, N, d = 1, 4, 1, 8 * 128 + 5, 128
    q, k, v = inputs.blasst_prefill_qkv(B, Hq, Hkv, N, d, "cpu", 32, sink_beta=2.0)
    lam = inputs.lambda_for(a, N)
    (dq, dk, dv), ref, st = _run(q, k, v, True, lam)
    assert (st == 1).sum() > 0                 # the case has skipped tiles
    _cmp(dq, ref["dq"], "dq")
    _cmp(dk, ref["dk"], "dk")
    _cmp(dv, ref["dv"], "dv")


def test_bwd_blasst_one_hot_sink():
    """With the workload's sink strength every row puts all of its weight on
    key 0 (P = 1 there to fp64 precision), so the exact dQ and dK vanish
    (the oracle's are ~1e-24) and a tolerance relative to their own size
    means nothing: check dV as usual and that dQ and dK are zero up to
    rounding, measured against dV's size."""
    B, Hq, Hkv, N, d = 1, 4, 1, 8 * 128 + 5, 128
    q, k, v = inputs.blasst_prefill_qkv(B, Hq, Hkv, N, d, "cpu", 32)
    (dq, dk, dv), ref, st = _run(q, k, v, True, inputs.lambda_for(10, N))
    assert (st == 1).sum() > 0
    _cmp(dv, ref["dv"], "dv")
    bound = 1e-5 * np.abs(ref["dv"]).max()
    assert np.abs(ref["dq"]).max() < bound and np.abs(ref["dk"]).max() < bound
    assert dq.float().abs().max().item() < bound, "dq"
    assert dk.float().abs().max().item() < bound, "dk"


def test_bwd_static_mask_with_empty_key_columns():
    """Per-head masks where key tile 2 is masked for every query tile: its
    dK and dV must be exactly zero."""
    B, Hq, Hkv, N, d = 1, 2, 2, 6 * 128, 64
    q, k, v = inputs.normal_qkv(B, Hq, Hkv, N, d, "cpu", 33)
    rng = np.random.default_rng(34)
    m = (rng.random((Hq, 6, 6)) < 0.6).astype(np.uint8)
    m[:, np.arange(6), np.arange(6)] = 1
    m[:, :, 2] = 0
    (dq, dk, dv), ref, _ = _run(q, k, v, False, 0.0, mask=m)
    _cmp(dq, ref["dq"], "dq")
    _cmp(dk, ref["dk"], "dk")
    _cmp(dv, ref["dv"], "dv")
    assert (dk[:, :, 256:384] == 0).all() and (dv[:, :, 256:384] == 0).all()


def test_bwd_varlen():
    """Key padding (three sequence lengths) on the BLASST recipe with the
    weaker sink, so that dQ and dK are not vanishingly small."""
    B, Hq, Hkv, N, d = 3, 2, 1, 4 * 128, 128
    q, k, v = inputs.blasst_prefill_qkv(B, Hq, Hkv, N, d, "cpu", 35, sink_beta=2.0)
    lens = [512, 300, 100]
    (dq, dk, dv), ref, _ = _run(q, k, v, True, inputs.lambda_for(10, N), seq_lens=lens)
    _cmp(dq, ref["dq"], "dq")
    _cmp(dk, ref["dk"], "dk")
    _cmp(dv, ref["dv"], "dv")
    for b, L in enumerate(lens):
        assert (dq[b, :, L:] == 0).all() and (dk[b, :, L:] == 0).all()
