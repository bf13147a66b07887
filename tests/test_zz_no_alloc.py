"""bsattn_fwd_decode_noalloc: the decode entry point for callers that cannot
allocate device memory (their framework owns all of it, or an allocation's
latency and failure are unacceptable on their path).  It must give the same
result as bsattn_fwd_decode with a caller-provided workspace, call after
call, and refuse problems that do not fit its fixed 32 MiB scratch.

This file is named so that pytest collects it last."""
import ctypes
import math

import pytest
import torch

from block_sparse_attention_bsattn_b200 import inputs
from tests.parity import compare_outputs

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20


def _ops():
    from block_sparse_attention_bsattn_b200 import ops
    return ops


@pytest.mark.parametrize("B,Hq,Hkv,L,splits,a", [(4, 8, 2, 4096 + 40, 4, 10.0),
                                                  (16, 32, 8, 16384, 16, 100.0)])
def test_noalloc_matches_workspace_decode_twice(B, Hq, Hkv, L, splits, a):
    ops = _ops()
    d, block = 128, 128
    q, k, v = inputs.blasst_decode_qkv(B, Hq, Hkv, L, d, "cuda", 2024 + B)
    lam = inputs.lambda_for(a, L)
    scale = 1 / math.sqrt(d)
    ref_o, ref_lse = ops.bsattn_fwd_decode(q, k, v, block, splits, scale, lam)
    torch.cuda.synchronize()
    ref_o_np = ref_o.float().cpu().numpy()
    ref_lse_np = ref_lse.cpu().numpy().astype("float64")
    for _ in range(2):
        o = torch.empty_like(q)
        lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        ops.bsattn_fwd_decode_noalloc(q, k, v, block, splits, o, scale, lam, lse=lse,
                                      status=status)
        torch.cuda.synchronize()
        assert status.item() == 0
        compare_outputs(o, ref_o_np, lse, ref_lse_np, "noalloc vs workspace decode")


def test_noalloc_rejects_problems_beyond_scratch():
    ops = _ops()
    # 64 x 64 x 16 x (128 + 2) x 4 bytes = 34 MB > 32 MiB
    B, Hq, d, splits = 64, 64, 128, 16
    assert ops.bsattn_decode_workspace_size(B, Hq, d, splits) > SCRATCH_BYTES
    P = ctypes.c_void_p
    rc = ops._lib.bsattn_fwd_decode_noalloc(P(0x1000), P(0x2000), P(0x3000), P(0x4000), None, B,
                                            Hq, 8, 4096, d, 128, 0.1, 0, 0.0, splits, None, None,
                                            None)
    assert rc == -4   # BSATTN_ERR_CAPACITY
