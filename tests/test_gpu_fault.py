"""Failure detection without a GPU fault: a test switch makes the prefill
kernels withhold their query tile (and the backward kernels their resident
tiles), so one pipeline wait runs out (a short limit).
The kernel must drain its own copies, free its tensor memory, return, and
report BSATTN_ERR_DEVICE_TIMEOUT in the status word; the context must stay
usable (a normal call afterwards is correct).  Nothing traps, faults or
hangs."""
import math

import pytest
import torch

import oracle
from block_sparse_attention_bsattn_b200 import inputs
from tests.parity import compare_outputs

pytestmark = pytest.mark.gpu


def _ops():
    from block_sparse_attention_bsattn_b200 import ops
    return ops


# two heads of one KV head (pair kernel, heads mode), one head (pair kernel,
# two consecutive query tiles), 64-token tiles and a block mask with one
# query head per KV head (one-query-tile kernel); lambda > 0 runs the
# variants with the skip vote, whose warps must all still meet at the vote
# barrier after the wait ran out
@pytest.mark.parametrize("hq,hkv,block,masked", [(2, 1, 128, False), (1, 1, 128, False),
                                                 (1, 1, 64, False), (2, 2, 128, True)])
@pytest.mark.parametrize("lam", [0.0, 1e-3])
def test_stalled_pipeline_reports_timeout_and_recovers(hq, hkv, block, masked, lam):
    ops = _ops()
    q, k, v = inputs.normal_qkv(1, hq, hkv, 256, 128, "cpu", 3)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    rp = ci = mask = None
    if masked:
        nb = 256 // block
        mask = torch.ones(1, nb, nb, dtype=torch.uint8)
        rp, ci, _ = ops.bsattn_build_index(mask.cuda(), block, block, True)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        ops.bsattn_debug_set(50_000_000, inject_stall=True)   # 50 ms per wait
        ops.bsattn_fwd_prefill(qd, kd, vd, block, None, True, lam, rp, ci, status=status)
        torch.cuda.synchronize()
        assert status.item() == -6, ops.bsattn_status_string(status.item())
    finally:
        ops.bsattn_debug_set(2_000_000_000, inject_stall=False)
    status.zero_()
    o, lse = ops.bsattn_fwd_prefill(qd, kd, vd, block, None, True, lam, rp, ci, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = oracle.prefill(q, k, v, block, 1 / math.sqrt(128), True, lam,
                         mask=None if mask is None else mask.numpy())
    compare_outputs(o, ref["o"], lse, ref["lse"], "after timeout")


@pytest.mark.parametrize("d,causal", [(128, True), (64, False)])
def test_backward_stall_reports_timeout_and_recovers(d, causal):
    """The backward kernels with their resident tiles withheld: the first
    wait of the MMA warp runs out, every role stops and drains, the status
    word says BSATTN_ERR_DEVICE_TIMEOUT, and the next call is correct."""
    ops = _ops()
    B, Hq, Hkv, N = 1, 4, 2, 3 * 128 + 17
    q, k, v = inputs.normal_qkv(B, Hq, Hkv, N, d, "cpu", 41)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    nq = -(-N // 128)
    st = torch.zeros(B, Hq, nq, nq, dtype=torch.uint8, device="cuda")
    o, lse = ops.bsattn_fwd_prefill(qd, kd, vd, 128, None, causal, 0.0, tile_status=st)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(42)).to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        ops.bsattn_debug_set(50_000_000, inject_stall=True)   # 50 ms per wait
        ops.bsattn_bwd_prefill(qd, kd, vd, o, dout.cuda(), lse, st, 128, None, causal,
                               status=status)
        torch.cuda.synchronize()
        assert status.item() == -6, ops.bsattn_status_string(status.item())
    finally:
        ops.bsattn_debug_set(2_000_000_000, inject_stall=False)
    status.zero_()
    dq, dk, dv = ops.bsattn_bwd_prefill(qd, kd, vd, o, dout.cuda(), lse, st, 128, None, causal,
                                        status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = oracle.prefill_bwd(q, k, v, dout, 128, 1 / math.sqrt(d), causal, st.cpu().numpy())
    for got, name in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        g = got.float().cpu().numpy()
        scale = max(abs(ref[name]).max(), 1e-6)
        assert abs(g - ref[name]).max() <= 3e-2 * scale, name
