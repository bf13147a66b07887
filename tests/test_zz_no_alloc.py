"""bsattn_fwd_decode_noalloc: the decode entry point for callers that cannot
allocate device memory (their framework owns all of it, or an allocation's
latency and failure are unacceptable on their path).  It must give the
result of bsattn_fwd_decode with a caller-provided workspace, and that of
the fp64 oracle, call after call, and refuse problems that do not fit its
fixed 32 MiB scratch.

This file is named so that pytest collects it last."""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_bsattn_b200 import inputs
from tests.parity import compare_outputs, compare_status

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20


def _ops():
    from block_sparse_attention_bsattn_b200 import ops
    return ops


# (B, Hq, Hkv, L, splits, a, oracle pairs): every (sequence, KV head) pair of
# the small case, eight spread over the larger one
CASES = [(4, 8, 2, 4096 + 40, 4, 10.0, None),
         (16, 32, 8, 16384, 16, 100.0, [(0, 0), (1, 7), (3, 2), (6, 5), (9, 1), (11, 6),
                                        (14, 3), (15, 4)])]


@pytest.mark.parametrize("B,Hq,Hkv,L,splits,a,pairs", CASES)
def test_noalloc_matches_workspace_decode_and_oracle_twice(B, Hq, Hkv, L, splits, a, pairs):
    ops = _ops()
    d, block = 128, 128
    T = -(-L // block)
    g = Hq // Hkv
    q, k, v = inputs.blasst_decode_qkv(B, Hq, Hkv, L, d, "cuda", 2024 + B)
    lam = inputs.lambda_for(a, L)
    scale = 1 / math.sqrt(d)
    ref_o, ref_lse = ops.bsattn_fwd_decode(q, k, v, block, splits, scale, lam)
    torch.cuda.synchronize()
    ref_o_np = ref_o.float().cpu().numpy()
    ref_lse_np = ref_lse.cpu().numpy().astype("float64")
    if pairs is None:
        pairs = [(b, h) for b in range(B) for h in range(Hkv)]
    qs, ks, vs = oracle.decode_problems(q.cpu(), k.cpu(), v.cpu(), pairs)
    orc = oracle.decode(qs, ks, vs, block, scale, lam, splits)
    for call in range(2):
        o = torch.empty_like(q)
        lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
        st = torch.zeros(B, Hkv, T, dtype=torch.uint8, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        ops.bsattn_fwd_decode_noalloc(q, k, v, block, splits, o, scale, lam, lse=lse,
                                      tile_status=st, status=status)
        torch.cuda.synchronize()
        assert status.item() == 0
        compare_outputs(o, ref_o_np, lse, ref_lse_np, f"call {call}: noalloc vs workspace decode")
        oc, lc, sc = o.float().cpu().numpy(), lse.cpu().numpy(), st.cpu().numpy()
        for p, (b, kvh) in enumerate(pairs):
            rows = slice(kvh * g, (kvh + 1) * g)
            what = f"call {call}: noalloc vs oracle, pair {(b, kvh)}"
            compare_outputs(oc[b, rows], orc["o"][p], lc[b, rows], orc["lse"][p], what)
            compare_status(sc[b, kvh], orc["status"][p], orc["margin"][p], what)
        assert np.isfinite(oc).all()


def test_noalloc_rejects_problems_beyond_scratch():
    ops = _ops()
    # 64 x 64 x 16 x (128 + 2) x 4 bytes = 34 MB > 32 MiB
    B, Hq, d, splits = 64, 64, 128, 16
    assert ops.bsattn_decode_workspace_size(B, Hq, d, splits) > SCRATCH_BYTES
    P = ctypes.c_void_p
    f = ops._lib.bsattn_fwd_decode_noalloc
    rc = f(P(0x1000), P(0x2000), P(0x3000), P(0x4000), None, B, Hq, 8, 4096, d, 128, 0.1, 0, 0.0,
           splits, None, None, None)
    assert rc == -4   # BSATTN_ERR_CAPACITY
    # argument errors are reported before the capacity
    assert f(None, P(0x2000), P(0x3000), P(0x4000), None, B, Hq, 8, 4096, d, 128, 0.1, 0, 0.0,
             splits, None, None, None) == -1
    assert f(P(0x1000), P(0x2000), P(0x3000), P(0x4000), None, B, Hq, 7, 4096, d, 128, 0.1, 0,
             0.0, splits, None, None, None) == -1
