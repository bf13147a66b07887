"""Index builder parity: bsattn_build_index against the oracle's CSR, bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_bsattn_b200 import inputs

pytestmark = pytest.mark.gpu


def _ops():
    from block_sparse_attention_bsattn_b200 import ops
    return ops


def _gpu_index(m, qb, kb, causal, capacity=None):
    ops = _ops()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rp, ci, nnz, order = ops.bsattn_build_index(torch.as_tensor(m).cuda().contiguous(), qb, kb,
                                                causal, capacity=capacity, status=status,
                                                with_order=True)
    torch.cuda.synchronize()
    rp, order = rp.cpu().numpy(), order.cpu().numpy()
    # the longest-first schedule: a stable sort of each head's rows by length
    Hm, nq = m.shape[0], m.shape[1]
    for h in range(Hm):
        lengths = np.diff(rp[h * (nq + 1):(h + 1) * (nq + 1)])
        expect = np.argsort(-lengths, kind="stable")
        assert (order[h * nq:(h + 1) * nq] == expect).all()
    return rp, ci.cpu().numpy(), nnz.cpu().numpy(), status.item()


@pytest.mark.parametrize("name", ["tiny", "mmdit", "videodit"])
@pytest.mark.parametrize("causal", [False, True])
def test_workload_masks(name, causal):
    m = {"tiny": inputs.mask_tiny, "mmdit": inputs.mask_mmdit,
         "videodit": inputs.mask_videodit}[name]().numpy()[None]
    rp, ci, nnz, st = _gpu_index(m, 128, 128, causal)
    rrp, rci, rnnz = oracle.build_index(m, 128, 128, causal)
    assert st == 0
    assert (rp == rrp).all() and (nnz == rnnz).all()
    assert (ci[: rnnz.sum()] == rci).all()


@pytest.mark.parametrize("heads,nq,nk", [(1, 1, 1), (3, 37, 70), (16, 300, 300), (2, 2100, 33)])
def test_random_masks(heads, nq, nk):
    rng = np.random.default_rng(heads * nq)
    m = (rng.random((heads, nq, nk)) < 0.3).astype(np.uint8)
    for causal in (False, True):
        rp, ci, nnz, st = _gpu_index(m, 64, 64, causal)
        rrp, rci, rnnz = oracle.build_index(m, 64, 64, causal)
        assert st == 0 and (rp == rrp).all() and (nnz == rnnz).all()
        assert (ci[: rnnz.sum()] == rci).all()


def test_causal_dense_count():
    m = np.ones((1, 256, 256), np.uint8)
    _, _, nnz, _ = _gpu_index(m, 128, 128, True)
    assert nnz.sum() == 32896


def test_capacity_overflow_reports_status():
    m = np.ones((1, 8, 8), np.uint8)
    rp, ci, nnz, st = _gpu_index(m, 64, 64, False, capacity=10)
    assert st == -4                      # BSATTN_ERR_CAPACITY
    assert nnz.sum() == 64 and rp[-1] == 64
