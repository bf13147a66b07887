"""Pins for the CPU oracle (no GPU).

Each test ties the oracle to something other than itself: the textbook dense
formula on special cases, brute force with an element mask, closed-form
two-tile examples of the BLASST skip rule, invariants (rows of the softmax
sum to one; a skipped tile contributes nothing; the executed set does not
depend on V), and the worked numbers printed on the pages.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_bsattn_b200 import inputs
from tests._refs import bf16_to_f64, dense_attention, element_mask


def _bf16(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


def _dense_ref(q, k, v, scale, block, causal, block_mask=None):
    """Per-head textbook reference with GQA (kv = h // g)."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    q64, k64, v64 = bf16_to_f64(q), bf16_to_f64(k), bf16_to_f64(v)
    out = np.zeros((B, Hq, N, d))
    lse = np.zeros((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            bm = np.ones((-(-N // block),) * 2, bool) if block_mask is None else \
                block_mask[0 if block_mask.shape[0] == 1 else h]
            allowed = element_mask(bm, block, N, causal)
            out[b, h], lse[b, h] = dense_attention(q64[b, h], k64[b, h // g], v64[b, h // g],
                                                   scale, allowed)
    return out, lse


# --------------------------------------------------------------- dense special cases
@pytest.mark.parametrize("B,Hq,Hkv,N,d,block,causal", [
    (1, 2, 2, 256, 64, 64, False),
    (2, 4, 2, 200, 64, 64, True),      # GQA g=2, ragged tail, causal
    (1, 4, 1, 300, 128, 128, False),   # MQA, ragged tail
    (1, 2, 2, 384, 128, 128, True),
])
def test_lambda0_all_ones_equals_dense(B, Hq, Hkv, N, d, block, causal):
    """"Attention 的七十二变" section 1 / BLASST section 3.1.1: with lambda = 0
    and no block mask the method is plain softmax(QK^T/sqrt(d))V."""
    q, k, v = inputs.normal_qkv(B, Hq, Hkv, N, d, "cpu", 7)
    scale = 1.0 / math.sqrt(d)
    r = oracle.prefill(q, k, v, block, scale, causal, 0.0)
    ref_o, ref_lse = _dense_ref(q, k, v, scale, block, causal)
    assert np.abs(r["o"] - ref_o).max() < 1e-12
    assert np.abs(r["lse"] - ref_lse).max() < 1e-12
    # every causally allowed tile visited and executed
    nq = -(-N // block)
    allowed = np.tril(np.ones((nq, nq), bool)) if causal else np.ones((nq, nq), bool)
    assert (r["status"] == np.where(allowed, 2, 0)[None, None]).all()


def test_static_mask_equals_brute_force_element_mask():
    """"块稀疏Attention实战" section 2.1: a zero block takes no part in QK,
    softmax or PV -- the same as -inf on every element of the block
    (section 5.2; the masked_fill reference of "Attention 的七十二变" 2.2).
    Tiny workload: B1 H2 N512 d64 block 64, diagonal +-1 plus block 0 global."""
    w = inputs.workload("tiny")
    r = oracle.prefill(w.q, w.k, w.v, w.block, w.scale, w.causal, 0.0, mask=w.mask.numpy())
    ref_o, ref_lse = _dense_ref(w.q, w.k, w.v, w.scale, w.block, False, w.mask.numpy())
    assert np.abs(r["o"] - ref_o).max() < 1e-12
    assert np.abs(r["lse"] - ref_lse).max() < 1e-12
    assert ((r["status"][0, 0] == 2) == (w.mask.numpy()[0] == 1)).all()


def test_static_mask_causal_per_head_mask_gqa():
    rng = np.random.default_rng(3)
    B, Hq, Hkv, N, d, block = 1, 4, 2, 320, 64, 64
    nq = -(-N // block)
    bm = (rng.random((Hq, nq, nq)) < 0.5).astype(np.uint8)
    bm[:, np.arange(nq), np.arange(nq)] = 1
    q, k, v = inputs.normal_qkv(B, Hq, Hkv, N, d, "cpu", 11)
    r = oracle.prefill(q, k, v, block, 0.125, True, 0.0, mask=bm)
    ref_o, ref_lse = _dense_ref(q, k, v, 0.125, block, True, bm)
    assert np.abs(r["o"] - ref_o).max() < 1e-12


def test_empty_mask_row_gives_zero_and_neg_inf():
    q, k, v = inputs.normal_qkv(1, 1, 1, 128, 64, "cpu", 5)
    bm = np.array([[[1, 0], [0, 0]]], np.uint8)
    r = oracle.prefill(q, k, v, 64, 0.125, False, 0.0, mask=bm)
    assert (r["o"][0, 0, 64:] == 0).all()
    assert np.isneginf(r["lse"][0, 0, 64:]).all()
    assert (r["status"][0, 0, 1] == 0).all()


# --------------------------------------------------------------- invariants
def test_rows_sum_to_one_with_blasst():
    """Softmax weights of every row sum to 1: with V = 1 the output is 1."""
    w = inputs.workload("blasst_prefill", shrink=True)
    v1 = torch.ones_like(w.v)
    for lam in (0.0, inputs.lambda_for(10, w.N), 1e-2):
        r = oracle.prefill(w.q, w.k, v1, w.block, w.scale, True, lam)
        assert np.abs(r["o"] - 1.0).max() < 1e-12


def test_skipped_tiles_contribute_nothing():
    """BLASST section 3.1.2: a skipped tile does no exp, no rowsum and no PV,
    so the result equals attention with that tile's keys removed (a static
    mask without the skipped tiles, lambda = 0)."""
    w = inputs.workload("blasst_prefill", shrink=True)
    lam = inputs.lambda_for(100, w.N)
    r = oracle.prefill(w.q, w.k, w.v, w.block, w.scale, True, lam)
    st = r["status"][0]                       # [Hq, nq, nk]
    assert (st == 1).sum() > 0, "workload should skip some tiles"
    keep = (st == 2).astype(np.uint8)         # per-head static mask
    r2 = oracle.prefill(w.q, w.k, w.v, w.block, w.scale, True, 0.0, mask=keep)
    assert np.abs(r["o"] - r2["o"]).max() < 1e-12
    assert np.abs(r["lse"] - r2["lse"]).max() < 1e-12


def test_executed_set_independent_of_v():
    w = inputs.workload("blasst_prefill", shrink=True)
    lam = inputs.lambda_for(10, w.N)
    r1 = oracle.prefill(w.q, w.k, w.v, w.block, w.scale, True, lam)
    r2 = oracle.prefill(w.q, w.k, torch.randn_like(w.v, dtype=torch.float32).to(torch.bfloat16),
                        w.block, w.scale, True, lam)
    assert (r1["status"] == r2["status"]).all()


def test_first_visited_tile_never_skipped_and_status_consistent():
    w = inputs.workload("blasst_prefill", shrink=True)
    r = oracle.prefill(w.q, w.k, w.v, w.block, w.scale, True, 1.0)
    st, mg = r["status"][0], r["margin"][0]
    assert (st[:, :, 0] == 2).all()
    vis = st > 0
    assert ((st == 1) == (vis & (mg < 0))).all()
    assert (st[:, :, 0] == 2).all() and np.isinf(mg[:, :, 0]).all()


# --------------------------------------------------------------- closed forms
def _two_tile_case(x, neg_row=None, swap=False):
    """N=128, block 64, d=64, H=1, scale 1.  Every query row is e0.  Tile 0:
    key 0 = 10 e0, keys 1..63 = 0.  Tile 1: every key = x e0.  (swap puts
    tile 1's keys first.)  Returns q, k, v as bf16 tensors."""
    N, d = 128, 64
    q = np.zeros((N, d)); q[:, 0] = 1.0
    if neg_row is not None:
        q[neg_row, 0] = -1.0
    k = np.zeros((N, d)); k[0, 0] = 10.0; k[64:, 0] = x
    if swap:
        k = np.concatenate([k[64:], k[:64]])
    rng = np.random.default_rng(0)
    v = np.round(rng.standard_normal((N, d)) * 8) / 8     # exact in bf16
    return (_bf16(q)[None, None], _bf16(k)[None, None], _bf16(v)[None, None], v)


def test_closed_form_skip():
    """BLASST section 3.1.1 with lambda = e^-5: tile 1's max (2) is 8 below the
    running max (10), 2 - 10 < -5, so it is skipped for every row and
    O = (e^10 v0 + sum_{k=1..63} v_k) / (e^10 + 63)."""
    q, k, v, v64 = _two_tile_case(2.0)
    r = oracle.prefill(q, k, v, 64, 1.0, False, math.exp(-5))
    assert (r["status"][0, 0, :, 1] == 1).all() and (r["status"][0, 0, :, 0] == 2).all()
    expect = (math.exp(10) * v64[0] + v64[1:64].sum(0)) / (math.exp(10) + 63)
    assert np.abs(r["o"][0, 0] - expect[None]).max() < 1e-12
    assert np.abs(r["lse"][0, 0] - math.log(math.exp(10) + 63)).max() < 1e-12
    np.testing.assert_allclose(r["margin"][0, 0, :, 1], -8.0 + 5.0, atol=1e-12)


def test_closed_form_keep():
    """x = 6: 6 - 10 = -4 > -5, tile kept:
    O = (e^10 v0 + sum_{1..63} v_k + e^6 sum_{64..127} v_k) / (e^10 + 63 + 64 e^6)."""
    q, k, v, v64 = _two_tile_case(6.0)
    r = oracle.prefill(q, k, v, 64, 1.0, False, math.exp(-5))
    assert (r["status"][0, 0] == 2).all()
    z = math.exp(10) + 63 + 64 * math.exp(6)
    expect = (math.exp(10) * v64[0] + v64[1:64].sum(0) + math.exp(6) * v64[64:].sum(0)) / z
    assert np.abs(r["o"][0, 0] - expect[None]).max() < 1e-12
    np.testing.assert_allclose(r["margin"][0, 0, :, 1], 1.0, atol=1e-12)


def test_closed_form_one_row_disagrees_keeps_tile():
    """All rows of the query tile must pass (the VOTE of the kernel design
    section).  Row 5 = -e0 sees tile-0 max 0 and tile-1 max -2: -2 > -5, so
    the tile is kept for the whole query tile 0; query tile 1 (rows 64..127,
    all e0) still skips it."""
    q, k, v, v64 = _two_tile_case(2.0, neg_row=5)
    r = oracle.prefill(q, k, v, 64, 1.0, False, math.exp(-5))
    assert r["status"][0, 0, 0, 1] == 2
    assert r["status"][0, 0, 1, 1] == 1
    # row 5 itself: scores tile0 = [-10, 0 x63], tile1 = [-2 x64]
    z = math.exp(-10) + 63 + 64 * math.exp(-2)
    expect = (math.exp(-10) * v64[0] + v64[1:64].sum(0) + math.exp(-2) * v64[64:].sum(0)) / z
    assert np.abs(r["o"][0, 0, 5] - expect).max() < 1e-12


def test_closed_form_order_matters():
    """Swapping the tiles: the big key is now in tile 1, whose max exceeds the
    running max, so nothing is skipped (tiles are visited in ascending order)."""
    q, k, v, v64 = _two_tile_case(2.0, swap=True)
    r = oracle.prefill(q, k, v, 64, 1.0, False, math.exp(-5))
    assert (r["status"][0, 0] == 2).all()


def test_closed_form_reverse_order():
    """Block-row reordering (the BLASST page's ablation, Figure 8): the tiles of
    a row are visited in descending order.  With the big key in tile 1, tile 1
    now sets the running max (10) and tile 0, whose max is 2, falls 8 below
    it: skipped, and O = (e^10 v64 + sum_{k=65..127} v_k) / (e^10 + 63).  With
    the big key in tile 0, reverse order keeps both tiles (tile 0's max is 8
    above tile 1's)."""
    q, k, v, v64 = _two_tile_case(2.0, swap=True)
    r = oracle.prefill(q, k, v, 64, 1.0, False, math.exp(-5), reverse=True)
    assert (r["status"][0, 0, :, 0] == 1).all() and (r["status"][0, 0, :, 1] == 2).all()
    expect = (math.exp(10) * v64[64] + v64[65:].sum(0)) / (math.exp(10) + 63)
    assert np.abs(r["o"][0, 0] - expect[None]).max() < 1e-12
    assert np.abs(r["lse"][0, 0] - math.log(math.exp(10) + 63)).max() < 1e-12
    np.testing.assert_allclose(r["margin"][0, 0, :, 0], -8.0 + 5.0, atol=1e-12)
    q, k, v, _ = _two_tile_case(2.0)
    r = oracle.prefill(q, k, v, 64, 1.0, False, math.exp(-5), reverse=True)
    assert (r["status"][0, 0] == 2).all()


def test_reverse_order_changes_nothing_without_skip():
    """With lambda = 0 the visit order only changes the summation order: the
    same visited tiles, every one executed, and the same O and LSE."""
    q, k, v = inputs.blasst_prefill_qkv(1, 2, 1, 3 * 64 + 17, 64, "cpu", 11)
    for causal in (False, True):
        a = oracle.prefill(q, k, v, 64, 0.125, causal, 0.0)
        b = oracle.prefill(q, k, v, 64, 0.125, causal, 0.0, reverse=True)
        assert (a["status"] == b["status"]).all() and (a["status"] != 1).all()
        assert np.abs(a["o"] - b["o"]).max() < 1e-12
        assert np.abs(a["lse"] - b["lse"]).max() < 1e-12


def test_reverse_order_with_mask_and_causal_first_tile_is_diagonal():
    """Reverse order over a block mask: the first visited tile of every row is
    its highest-index allowed tile, which is never skipped."""
    rng = np.random.default_rng(5)
    nb, block = 5, 64
    N = nb * block - 9
    m = (rng.random((1, nb, nb)) < 0.5).astype(np.uint8)
    m[0, np.arange(nb), np.arange(nb)] = 1
    q, k, v = inputs.blasst_prefill_qkv(1, 1, 1, N, 64, "cpu", 12)
    r = oracle.prefill(q, k, v, block, 0.125, True, 0.5, mask=m, reverse=True)
    for i in range(nb):
        allowed = [j for j in range(nb) if m[0, i, j] and j <= i]
        assert r["status"][0, 0, i, max(allowed)] == 2
        assert set(np.nonzero(r["status"][0, 0, i])[0]) == set(allowed)


def test_lambda_zero_and_one_edges():
    q, k, v, _ = _two_tile_case(2.0)
    r0 = oracle.prefill(q, k, v, 64, 1.0, False, 0.0)
    assert (r0["status"][0, 0] == 2).all()
    # lambda = 1 (ln = 0): skip iff the tile max is below the running max
    r1 = oracle.prefill(q, k, v, 64, 1.0, False, 1.0)
    assert (r1["status"][0, 0, :, 1] == 1).all()
    q2, k2, v2, _ = _two_tile_case(10.0)      # tile 1 max ties the running max
    r2 = oracle.prefill(q2, k2, v2, 64, 1.0, False, 1.0)
    assert (r2["status"][0, 0, :, 1] == 2).all()
    with pytest.raises(oracle.OracleError):
        oracle.prefill(q, k, v, 64, 1.0, False, 1.5)


def test_causal_tile_visits():
    w = inputs.workload("blasst_prefill", shrink=True)
    r = oracle.prefill(w.q, w.k, w.v, w.block, w.scale, True, 0.0)
    nq = w.nq
    assert (r["status"][0, 0] > 0).sum() == nq * (nq + 1) // 2


# --------------------------------------------------------------- decode
def test_decode_lambda0_equals_dense():
    w = inputs.workload("blasst_decode", shrink=True)
    pairs = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    qs, ks, vs = oracle.decode_problems(w.q, w.k, w.v, pairs)
    r = oracle.decode(qs, ks, vs, w.block, w.scale, 0.0, w.num_splits)
    q64, k64, v64 = bf16_to_f64(qs), bf16_to_f64(ks), bf16_to_f64(vs)
    for p in range(len(pairs)):
        o, lse = dense_attention(q64[p], k64[p], v64[p], w.scale)
        assert np.abs(r["o"][p] - o).max() < 1e-12
        assert np.abs(r["lse"][p] - lse).max() < 1e-12
    assert (r["status"] == 2).all()


def test_decode_equals_prefill_row_for_single_split():
    """With one split, the decode query tile (the g heads of a KV head) is the
    prefill algorithm applied to g query rows that all sit after every key."""
    rng = np.random.default_rng(9)
    g, L, d, block = 4, 640, 64, 64
    q = _bf16(rng.standard_normal((1, g, d)))
    k = _bf16(rng.standard_normal((1, L, d)) + 3 * rng.standard_normal((1, L // 64, 1, d)).repeat(64, 1).reshape(1, L, d))
    v = _bf16(rng.standard_normal((1, L, d)))
    lam = 0.05
    r = oracle.decode(q, k, v, block, 0.125, lam, 1)
    # prefill form: append the g queries as the rows of one extra (last) tile
    q_full = torch.zeros(1, 1, L + block, d, dtype=torch.bfloat16)
    k_full = torch.zeros(1, 1, L + block, d, dtype=torch.bfloat16)
    v_full = torch.zeros(1, 1, L + block, d, dtype=torch.bfloat16)
    q_full[0, 0, L:L + g] = q[0]
    k_full[0, 0, :L] = k[0]
    v_full[0, 0, :L] = v[0]
    nt = L // block
    bm = np.zeros((1, nt + 1, nt + 1), np.uint8)
    bm[0, nt, :nt] = 1
    rp = oracle.prefill(q_full[:, :, :L + g].contiguous(), k_full[:, :, :L + g].contiguous(),
                        v_full[:, :, :L + g].contiguous(), block, 0.125, False, lam, mask=bm)
    assert np.abs(rp["o"][0, 0, L:L + g] - r["o"][0]).max() < 1e-12
    assert (rp["status"][0, 0, nt, :nt] == r["status"][0]).all()


def test_decode_split_resets_running_max():
    """Reading of split-KV: the running max restarts at -inf in each split, so
    the first tile of every split is executed even when an earlier split
    already holds a far larger score."""
    g, d, block = 1, 64, 64
    L = 4 * block
    q = np.zeros((1, g, d)); q[0, 0, 0] = 1.0
    k = np.zeros((1, L, d)); k[0, 0, 0] = 20.0          # huge score in tile 0
    v = np.random.default_rng(1).integers(-4, 5, (1, L, d)).astype(np.float64)
    lam = math.exp(-5)
    one = oracle.decode(_bf16(q), _bf16(k), _bf16(v), block, 1.0, lam, 1)
    assert list(one["status"][0]) == [2, 1, 1, 1]
    two = oracle.decode(_bf16(q), _bf16(k), _bf16(v), block, 1.0, lam, 2)
    # split 2 restarts at tile 2: its max (0) passes nothing, and tile 3 ties it
    assert list(two["status"][0]) == [2, 1, 2, 2]
    # closed form for two splits: tiles 0, 2 and 3 executed
    s = np.concatenate([[20.0], np.zeros(63), np.zeros(128)])
    vv = np.concatenate([v[0, :64], v[0, 128:256]])
    p = np.exp(s - 20.0)
    assert np.abs(two["o"][0, 0] - (p @ vv) / p.sum()).max() < 1e-12


def test_decode_sink_seed_closed_form():
    """Sink seeding: every split after the first starts its running max from
    key tile 0's row max.  Tile 0 holds a score of 10 (the sink), tiles 2 and 3
    scores of 2.  Unseeded, split 2 restarts at -inf and executes both of its
    tiles; seeded, both fall 8 below the sink (2 - 10 < -5) and are skipped,
    leaving O = (e^10 v0 + sum_{k=1..63} v_k) / (e^10 + 63)."""
    g, d, block = 1, 64, 64
    L = 4 * block
    q = np.zeros((1, g, d)); q[0, 0, 0] = 1.0
    k = np.zeros((1, L, d)); k[0, 0, 0] = 10.0; k[0, 2 * block:, 0] = 2.0
    v = np.random.default_rng(2).integers(-4, 5, (1, L, d)).astype(np.float64)
    lam = math.exp(-5)
    plain = oracle.decode(_bf16(q), _bf16(k), _bf16(v), block, 1.0, lam, 2)
    assert list(plain["status"][0]) == [2, 1, 2, 2]
    seeded = oracle.decode(_bf16(q), _bf16(k), _bf16(v), block, 1.0, lam, 2, sink_seed=True)
    assert list(seeded["status"][0]) == [2, 1, 1, 1]
    expect = (math.exp(10) * v[0, 0] + v[0, 1:64].sum(0)) / (math.exp(10) + 63)
    assert np.abs(seeded["o"][0, 0] - expect).max() < 1e-12
    np.testing.assert_allclose(seeded["margin"][0, 2:], [-3.0, -3.0], atol=1e-12)
    # one split: seeding has nothing to seed
    one_p = oracle.decode(_bf16(q), _bf16(k), _bf16(v), block, 1.0, lam, 1)
    one_s = oracle.decode(_bf16(q), _bf16(k), _bf16(v), block, 1.0, lam, 1, sink_seed=True)
    assert (one_p["status"] == one_s["status"]).all()
    assert np.abs(one_p["o"] - one_s["o"]).max() == 0.0


def test_decode_sink_seed_only_adds_skips():
    """A seeded running max is never below the unseeded one, so seeding can
    only turn executed tiles into skipped ones; with lambda = 0 it changes
    nothing."""
    q, k, v = inputs.blasst_decode_qkv(2, 8, 2, 40 * 64 + 5, 64, "cpu", 13)
    qs, ks, vs = oracle.decode_problems(q, k, v, [(0, 0), (0, 1), (1, 0), (1, 1)])
    a = oracle.decode(qs, ks, vs, 64, 0.125, 1e-2, 5)
    b = oracle.decode(qs, ks, vs, 64, 0.125, 1e-2, 5, sink_seed=True)
    assert ((b["status"] == 2) <= (a["status"] == 2)).all()
    assert (b["status"] == 1).sum() > (a["status"] == 1).sum()
    a0 = oracle.decode(qs, ks, vs, 64, 0.125, 0.0, 5)
    b0 = oracle.decode(qs, ks, vs, 64, 0.125, 0.0, 5, sink_seed=True)
    assert (a0["status"] == b0["status"]).all()
    assert np.abs(a0["o"] - b0["o"]).max() == 0.0


@pytest.mark.parametrize("causal,masked,lam", [(True, False, 0.0), (True, False, 2e-2),
                                               (False, True, 1e-2), (True, True, 5e-2)])
def test_varlen_prefill_equals_each_sequence_alone(causal, masked, lam):
    """Key padding (the multimodal DiT page, section 5.2): a batch padded to
    N with valid lengths len_b gives, for every sequence, exactly what the
    sequence gives alone at N = len_b (same O, LSE, executed tiles), and its
    padding rows get O = 0 and LSE = -inf."""
    B, Hq, Hkv, N, d, block = 4, 4, 2, 5 * 64 + 9, 64, 64
    lens = [N, 200, 64, 0]
    q, k, v = inputs.blasst_prefill_qkv(B, Hq, Hkv, N, d, "cpu", 17)
    nb = -(-N // block)
    mask = None
    if masked:
        rng = np.random.default_rng(4)
        mask = (rng.random((1, nb, nb)) < 0.6).astype(np.uint8)
        mask[0, np.arange(nb), np.arange(nb)] = 1
    r = oracle.prefill(q, k, v, block, 0.125, causal, lam, mask=mask, seq_lens=lens)
    for b, L in enumerate(lens):
        if L > 0:
            nl = -(-L // block)
            m = None if mask is None else np.ascontiguousarray(mask[:, :nl, :nl])
            alone = oracle.prefill(q[b:b + 1, :, :L], k[b:b + 1, :, :L], v[b:b + 1, :, :L], block,
                                   0.125, causal, lam, mask=m)
            assert np.abs(r["o"][b, :, :L] - alone["o"][0]).max() < 1e-12
            assert np.abs(r["lse"][b, :, :L] - alone["lse"][0]).max() < 1e-12
            assert (r["status"][b, :, :nl, :nl] == alone["status"][0]).all()
            assert (r["status"][b, :, :, nl:] == 0).all() and (r["status"][b, :, nl:] == 0).all()
        assert (r["o"][b, :, L:] == 0).all()
        assert np.isneginf(r["lse"][b, :, L:]).all()


def test_varlen_decode_equals_each_cache_alone():
    """Decode with per-sequence cache lengths: each problem equals its cache
    truncated to its own length, split by the same num_splits."""
    n, g, L, d, block = 5, 4, 23 * 64 + 7, 64, 64
    lens = [L, 1000, 64, 1, 0]
    q, k, v = inputs.blasst_decode_qkv(1, n * g, n, L, d, "cpu", 18)
    qs, ks, vs = oracle.decode_problems(q, k, v, [(0, x) for x in range(n)])
    for seed in (False, True):
        r = oracle.decode(qs, ks, vs, block, 0.125, 1e-2, 4, sink_seed=seed, lens=lens)
        for p, Lp in enumerate(lens):
            if Lp == 0:
                assert (r["o"][p] == 0).all() and np.isneginf(r["lse"][p]).all()
                assert (r["status"][p] == 0).all()
                continue
            alone = oracle.decode(qs[p:p + 1], ks[p:p + 1, :Lp], vs[p:p + 1, :Lp], block, 0.125,
                                  1e-2, 4, sink_seed=seed)
            Tp = -(-Lp // block)
            assert np.abs(r["o"][p] - alone["o"][0]).max() < 1e-12
            assert np.abs(r["lse"][p] - alone["lse"][0]).max() < 1e-12
            assert (r["status"][p, :Tp] == alone["status"][0]).all()
            assert (r["status"][p, Tp:] == 0).all()
    # closed form: a cache of 4 tiles inside a buffer of 8, two splits.  Its own
    # tiles split {0, 1} {2, 3}: tile 2 starts a split and is executed, and
    # tile 3 ties it; the buffer's tiles would have split {0..3} and skipped
    # tiles 1..3 (score 0, 10 below key 0's)
    d1, blk = 64, 64
    q1 = np.zeros((1, 1, d1)); q1[0, 0, 0] = 1.0
    k1 = np.zeros((1, 8 * blk, d1)); k1[0, 0, 0] = 10.0
    v1 = np.random.default_rng(5).integers(-4, 5, (1, 8 * blk, d1)).astype(np.float64)
    r1 = oracle.decode(_bf16(q1), _bf16(k1), _bf16(v1), blk, 1.0, math.exp(-5), 2, lens=[4 * blk])
    assert list(r1["status"][0]) == [2, 1, 2, 2, 0, 0, 0, 0]


def test_decode_gqa_group_vote():
    """Decode query tile = the g query heads of one KV head; a V tile is skipped
    only when all g heads pass."""
    d, block, L = 64, 64, 128
    q = np.zeros((1, 2, d)); q[0, 0, 0] = 1.0; q[0, 1, 0] = -1.0
    k = np.zeros((1, L, d)); k[0, 0, 0] = 10.0; k[0, 64:, 0] = 2.0
    v = np.ones((1, L, d))
    r = oracle.decode(_bf16(q), _bf16(k), _bf16(v), block, 1.0, math.exp(-5), 1)
    assert list(r["status"][0]) == [2, 2]
    r1 = oracle.decode(_bf16(q[:, :1]), _bf16(k), _bf16(v), block, 1.0, math.exp(-5), 1)
    assert list(r1["status"][0]) == [2, 1]


# --------------------------------------------------------------- index
def test_index_matches_definition_and_causal():
    rng = np.random.default_rng(5)
    m = (rng.random((3, 9, 9)) < 0.4).astype(np.uint8)
    for causal in (False, True):
        rp, ci, nnz = oracle.build_index(m, 64, 64, causal)
        pos = 0
        for h in range(3):
            for i in range(9):
                cols = [j for j in range(9) if m[h, i, j] and (not causal or j <= i)]
                assert rp[h * 10 + i] == pos
                assert list(ci[pos:pos + len(cols)]) == cols
                pos += len(cols)
            assert rp[h * 10 + 9] == pos
        assert nnz.sum() == pos
    with pytest.raises(oracle.OracleError):
        oracle.build_index(m, 64, 64, False, capacity=3)
