"""Decode parity: bsattn_fwd_decode (split kernel + combine, through the C ABI)
against the fp64 oracle on the same seeded inputs."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_bsattn_b200 import inputs
from tests.parity import compare_outputs, compare_status

pytestmark = pytest.mark.gpu


def _ops():
    from block_sparse_attention_bsattn_b200 import ops
    return ops


def _run(q, k, v, block, splits, scale, lam, sink_seed=False):
    ops = _ops()
    B, Hq, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    T = -(-L // block)
    st = torch.zeros(B, Hkv, T, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = ops.bsattn_fwd_decode(q.cuda(), k.cuda(), v.cuda(), block, splits, scale, lam,
                                   tile_status=st, status=status, sink_seed=sink_seed)
    torch.cuda.synchronize()
    assert status.item() == 0, ops.bsattn_status_string(status.item())
    return o, lse, st


def _check(q, k, v, block, splits, scale, lam, pairs=None, what="", sink_seed=False):
    o, lse, st = _run(q, k, v, block, splits, scale, lam, sink_seed)
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    if pairs is None:
        pairs = [(b, h) for b in range(B) for h in range(Hkv)]
    qs, ks, vs = oracle.decode_problems(q, k, v, pairs)
    ref = oracle.decode(qs.cpu(), ks.cpu(), vs.cpu(), block, scale, lam, splits,
                        sink_seed=sink_seed)
    o_c, lse_c, st_c = o.float().cpu().numpy(), lse.cpu().numpy(), st.cpu().numpy()
    for p, (b, kvh) in enumerate(pairs):
        compare_outputs(o_c[b, kvh * g:(kvh + 1) * g], ref["o"][p], lse_c[b, kvh * g:(kvh + 1) * g],
                        ref["lse"][p], f"{what} pair {(b, kvh)}")
        compare_status(st_c[b, kvh], ref["status"][p], ref["margin"][p], f"{what} pair {(b, kvh)}")
    return ref


@pytest.mark.parametrize("a", inputs.A_SWEEP)
def test_blasst_decode_shrunk(a):
    w = inputs.workload("blasst_decode", shrink=True)
    _check(w.q, w.k, w.v, w.block, w.num_splits, w.scale, inputs.lambda_for(a, w.N), what=f"a={a}")


def test_decode_operating_point_shrunk():
    """The benchmark's decode operating point (4 splits, a = 160: the BLASST
    page's 73.2% decode sparsity on this recipe) on the shrunk workload."""
    w = inputs.workload("blasst_decode", shrink=True)
    _check(w.q, w.k, w.v, w.block, inputs.DECODE_OP_SPLITS, w.scale,
           inputs.lambda_for(inputs.DECODE_OP_A, w.N), what="operating point")


@pytest.mark.parametrize("d,block,g", [(64, 64, 1), (64, 128, 2), (128, 64, 8), (128, 128, 4),
                                       (128, 128, 8), (128, 128, 3), (64, 128, 16),
                                       (128, 128, 1), (128, 128, 16), (128, 128, 5),
                                       (64, 128, 6), (128, 128, 12), (128, 64, 16),
                                       (64, 64, 3), (128, 64, 5), (64, 64, 12)])
@pytest.mark.parametrize("splits", [1, 3, 7])
def test_decode_shapes(d, block, g, splits):
    B, Hkv, L = 2, 2, 5 * block + 19
    q, k, v = inputs.blasst_decode_qkv(B, Hkv * g, Hkv, L, d, "cpu", 31 + d + g)
    _check(q, k, v, block, splits, 1 / math.sqrt(d), 2e-3, what=f"d{d} b{block} g{g} s{splits}")


@pytest.mark.parametrize("a", [0.0, 10.0, 1000.0])
def test_decode_table4_shape_shrunk(a):
    """32 query / 4 KV heads (group of 8), the BLASST page's Table 4 decode shape
    with fewer sequences and a shorter cache."""
    q, k, v = inputs.blasst_decode_qkv(3, 32, 4, 8192, 128, "cpu", 4243)
    _check(q, k, v, 128, 16, 1 / math.sqrt(128), inputs.lambda_for(a, 8192), what=f"t4 a={a}")


@pytest.mark.parametrize("d,block,g", [(128, 128, 4), (128, 128, 8), (64, 128, 3),
                                       (128, 64, 4), (64, 64, 1)])
def test_sink_seeded_splits(d, block, g):
    """Splits after the first start their running max from key tile 0's row
    max: both decode kernels against the oracle's seeded splits, and more V
    tiles skipped than without seeding."""
    B, Hkv, L = 2, 2, 23 * block + 7
    q, k, v = inputs.blasst_decode_qkv(B, Hkv * g, Hkv, L, d, "cpu", 57 + g + block)
    lam = inputs.lambda_for(10.0, L)
    seeded = _check(q, k, v, block, 5, 1 / math.sqrt(d), lam, what=f"seed d{d} b{block} g{g}",
                    sink_seed=True)
    plain = _check(q, k, v, block, 5, 1 / math.sqrt(d), lam, what="plain")
    assert (seeded["status"] == 1).sum() > (plain["status"] == 1).sum()


def test_sink_seed_with_empty_splits():
    q, k, v = inputs.blasst_decode_qkv(1, 4, 1, 300, 128, "cpu", 9)
    _check(q, k, v, 128, 8, 1 / math.sqrt(128), 1e-2, what="seeded empty splits", sink_seed=True)


@pytest.mark.parametrize("d,block,g", [(128, 128, 4), (64, 128, 8), (128, 64, 4), (64, 64, 2)])
@pytest.mark.parametrize("sink_seed", [False, True])
def test_varlen_cache_lengths(d, block, g, sink_seed):
    """Per-sequence cache lengths: both decode kernels against the oracle's
    problems at their own lengths (splits cut each cache's own tiles)."""
    ops = _ops()
    B, Hkv, L, splits = 5, 2, 19 * block + 11, 4
    lens = [L, 7 * block + 3, block, 1, 0]
    q, k, v = inputs.blasst_decode_qkv(B, Hkv * g, Hkv, L, d, "cpu", 61 + g + block)
    lam = 1e-2
    T = -(-L // block)
    st = torch.zeros(B, Hkv, T, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o, lse = ops.bsattn_fwd_decode(q.cuda(), k.cuda(), v.cuda(), block, splits, 1 / math.sqrt(d),
                                   lam, tile_status=st, status=status, sink_seed=sink_seed,
                                   seq_lens=sl)
    torch.cuda.synchronize()
    assert status.item() == 0, ops.bsattn_status_string(status.item())
    pairs = [(b, h) for b in range(B) for h in range(Hkv)]
    qs, ks, vs = oracle.decode_problems(q, k, v, pairs)
    ref = oracle.decode(qs.cpu(), ks.cpu(), vs.cpu(), block, 1 / math.sqrt(d), lam, splits,
                        sink_seed=sink_seed, lens=[lens[b] for b, _ in pairs])
    o_c, lse_c, st_c = o.float().cpu().numpy(), lse.cpu().numpy(), st.cpu().numpy()
    for p_, (b, kvh) in enumerate(pairs):
        rows = slice(kvh * g, (kvh + 1) * g)
        compare_outputs(o_c[b, rows], ref["o"][p_], lse_c[b, rows], ref["lse"][p_],
                        f"varlen decode pair {(b, kvh)}")
        compare_status(st_c[b, kvh], ref["status"][p_], ref["margin"][p_], "varlen decode")
    assert (o_c[4] == 0).all() and np.isneginf(lse_c[4]).all()   # an empty cache


def test_long_cache():
    """A 1,048,699-token cache (8,193 tiles, 16 splits of 513) for one
    sequence and a GQA group of 4, against the oracle."""
    q, k, v = inputs.blasst_decode_qkv(1, 4, 1, (1 << 20) + 123, 128, "cuda", 77)
    _check(q, k, v, 128, 16, 1 / math.sqrt(128), inputs.lambda_for(10.0, (1 << 20) + 123),
           what="1M-token cache")


def test_more_splits_than_tiles():
    q, k, v = inputs.blasst_decode_qkv(1, 4, 1, 300, 128, "cpu", 9)
    _check(q, k, v, 128, 8, 1 / math.sqrt(128), 1e-2, what="empty splits")


@pytest.mark.parametrize("a", [0.0, 10.0])
def test_blasst_decode_full_size_sampled(a):
    """B64 Hq32/Hkv8 L131072 d128, 16 splits, in the launch configuration the
    benchmark times; 8 (batch, KV head) problems checked against the oracle."""
    w = inputs.workload("blasst_decode", device="cuda")
    rng = np.random.default_rng(17)
    pairs = sorted({(int(rng.integers(w.B)), int(rng.integers(w.Hkv))) for _ in range(8)})
    _check(w.q, w.k, w.v, w.block, w.num_splits, w.scale, inputs.lambda_for(a, w.N), pairs,
           what=f"full a={a}")


@pytest.mark.parametrize("lam", [1.0, 1e-30])
@pytest.mark.parametrize("block", [64, 128])
def test_decode_lambda_at_the_ends_of_its_range(lam, block):
    """lambda = 1 (a tile is skipped unless some query head reaches the
    running max) and lambda = 1e-30 (effectively no skipping)."""
    B, Hkv, g, L = 2, 2, 4, 9 * block + 11
    q, k, v = inputs.blasst_decode_qkv(B, Hkv * g, Hkv, L, 128, "cpu", 71 + block)
    ref = _check(q, k, v, block, 3, 1 / math.sqrt(128), lam, what=f"lambda {lam} b{block}")
    if lam == 1.0:
        assert (ref["status"] == 1).sum() > 0
