"""The exponential that the prefill kernels evaluate on the FMA and integer
pipes for part of a kept tile's columns, against 2^x in fp64 (its error
bound) and against the special-function unit's exp2 (torch.exp2 on the GPU)."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_fma_pipe_exp2_error_bound():
    from block_sparse_attention_bsattn_b200 import ops
    g = torch.Generator().manual_seed(5)
    x = torch.cat([torch.linspace(-126.0, 8.0, 1 << 20),
                   torch.rand(1 << 20, generator=g) * 8 - 4,             # the common range
                   torch.tensor([0.0, -0.0, 1.0, -1.0, 7.999999, 8.0, 63.5, -125.999])])
    y = ops.bsattn_debug_exp2(x.cuda()).cpu().double().numpy()
    ref = np.exp2(x.double().numpy())
    rel = np.abs(y - ref) / ref
    assert rel.max() < 1e-4, rel.max()
    # against the special-function unit's exp2 on the same inputs
    sfu = torch.exp2(x.cuda()).cpu().double().numpy()
    assert (np.abs(y - sfu) / sfu).max() < 2e-4
    # integers are exact (2^0 = 1 and so on)
    xi = torch.arange(-126, 64, dtype=torch.float32)
    assert torch.equal(ops.bsattn_debug_exp2(xi.cuda()).cpu(), torch.exp2(xi.double()).float())


def test_fma_pipe_exp2_underflow_and_odd_length():
    from block_sparse_attention_bsattn_b200 import ops
    x = torch.tensor([-127.0, -200.0, -1e30, float("-inf"), 0.5], device="cuda")
    y = ops.bsattn_debug_exp2(x).cpu()
    assert (y[:4] == 0).all()
    assert abs(y[4].item() / 2 ** 0.5 - 1) < 1e-4
    assert ops.bsattn_debug_exp2(torch.empty(0, device="cuda")).numel() == 0
