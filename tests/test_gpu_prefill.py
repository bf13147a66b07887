"""Prefill parity: the CUDA path (bsattn_build_index + bsattn_fwd_prefill
through the C ABI) against the fp64 oracle on the same seeded inputs."""
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


def _run_gpu(w, lam, mask=None, mask_heads=1, ordered=True, reverse=False, skip_v=False):
    """Index (with the longest-first row order unless `ordered` is False) and
    prefill through the C ABI; returns (o, lse, tile_status)."""
    ops = _ops()
    q, k, v = w.q.cuda(), w.k.cuda(), w.v.cuda()
    rp = ci = order = None
    if mask is not None:
        m = torch.as_tensor(mask, dtype=torch.uint8).cuda().contiguous()
        rp, ci, _, order = ops.bsattn_build_index(m, w.block, w.block, w.causal, with_order=True)
        mask_heads = m.shape[0]
        if not ordered:
            order = None
    st = torch.zeros(w.B, w.Hq, w.nq, w.nk, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = ops.bsattn_fwd_prefill(q, k, v, w.block, w.scale, w.causal, lam, rp, ci, mask_heads,
                                    tile_status=st, status=status, row_order=order,
                                    reverse=reverse, skip_v=skip_v)
    torch.cuda.synchronize()
    assert status.item() == 0, ops.bsattn_status_string(status.item())
    return o, lse, st


def _check(w, lam, mask=None, what="", ordered=True, reverse=False, skip_v=False):
    o, lse, st = _run_gpu(w, lam, mask, ordered=ordered, reverse=reverse, skip_v=skip_v)
    ref = oracle.prefill(w.q, w.k, w.v, w.block, w.scale, w.causal, lam, mask=mask,
                         reverse=reverse)
    compare_outputs(o, ref["o"], lse, ref["lse"], what)
    compare_status(st, ref["status"], ref["margin"], what)
    return ref


@pytest.mark.parametrize("name", ["tiny", "mmdit", "videodit"])
@pytest.mark.parametrize("ordered", [True, False])
def test_static_mask_workloads_shrunk(name, ordered):
    w = inputs.workload(name, shrink=True)
    _check(w, 0.0, w.mask.numpy(), name, ordered=ordered)


def test_mmdit_full_size():
    """Multimodal DiT at full size (B1 H24 N4352 d64 block 128): every output."""
    w = inputs.workload("mmdit")
    _check(w, 0.0, w.mask.numpy(), "mmdit")


@pytest.mark.parametrize("a", inputs.A_SWEEP)
def test_blasst_prefill_shrunk(a):
    w = inputs.workload("blasst_prefill", shrink=True)
    ref = _check(w, inputs.lambda_for(a, w.N), None, f"blasst a={a}")
    if a >= 10:
        assert (ref["status"] == 1).sum() > 0


@pytest.mark.parametrize("d,block", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("hq,hkv,nt", [(4, 1, 3), (3, 3, 4)])
def test_dense_shapes_and_tails(d, block, causal, hq, hkv, nt):
    """Every (d, block) variant, causal and not, with a ragged tail; GQA 4
    (head pairs share a CTA) and GQA 1 with an odd number of query tiles
    (consecutive query tiles share a CTA, the last one alone)."""
    B, Hq, Hkv, N = 2, hq, hkv, nt * block + 37
    q, k, v = inputs.normal_qkv(B, Hq, Hkv, N, d, "cpu", 100 + d + block)
    w = inputs.Workload("dense", B, Hq, Hkv, N, d, block, causal, "prefill", 1 / math.sqrt(d),
                        None, q=q, k=k, v=v)
    _check(w, 0.0, None, f"d{d} b{block} c{causal}")


@pytest.mark.parametrize("d,block", [(64, 64), (128, 128)])
def test_blasst_random_masks_per_head(d, block):
    """Per-head random static masks combined with the dynamic skip."""
    rng = np.random.default_rng(d + block)
    B, Hq, Hkv, N = 1, 4, 2, 6 * block - 5
    nb = -(-N // block)
    m = (rng.random((Hq, nb, nb)) < 0.6).astype(np.uint8)
    m[:, np.arange(nb), np.arange(nb)] = 1
    m[:, 2, :] = 0                                 # an empty row
    q, k, v = inputs.blasst_prefill_qkv(B, Hq, Hkv, N, d, "cpu", 7)
    w = inputs.Workload("rand", B, Hq, Hkv, N, d, block, True, "prefill", 1 / math.sqrt(d), None,
                        q=q, k=k, v=v)
    o, lse, st = _run_gpu(w, 3e-3, m)
    ref = oracle.prefill(q, k, v, block, w.scale, True, 3e-3, mask=m)
    compare_outputs(o, ref["o"], lse, ref["lse"])
    compare_status(st, ref["status"], ref["margin"])
    # the empty row: zeros and -inf
    rows = slice(2 * block, 3 * block)
    assert (o[:, :, rows].float() == 0).all()
    assert torch.isneginf(lse[:, :, rows]).all()


@pytest.mark.parametrize("d,block", [(64, 64), (128, 128)])
@pytest.mark.parametrize("lam", [0.0, 3e-3])
def test_running_max_jumps_in_a_later_tile(d, block, lam):
    """Scores that jump far beyond the lazy-rescale slack (8 in base 2) in a
    later key tile: in the low half of key tile 2's columns for the first half
    of the last query tile's rows, in the high half of key tile 3 for the
    rest.  The exponent shift then moves after the first kept tile, so the
    one-tile kernel's exponentials taken before the two column halves have
    exchanged their maxima must be redone for those rows (one query head per
    KV head, per-head all-ones masks: the one-tile kernel)."""
    B, Hq, Hkv, nt = 1, 2, 2, 5
    N = nt * block
    q, k, v = inputs.normal_qkv(B, Hq, Hkv, N, d, "cpu", 321 + d)
    scale = 1 / math.sqrt(d)
    qf, kf = q.float(), k.float()
    r0 = (nt - 1) * block
    for h in range(Hq):
        for r in range(block):
            key = (2 * block + r) if r < block // 2 else (3 * block + r)
            qr = qf[0, h, r0 + r]
            kf[0, h, key] = qr * (20.0 / (scale * float(qr @ qr)))   # score 20 for this row
    k = kf.to(torch.bfloat16)
    w = inputs.Workload("jump", B, Hq, Hkv, N, d, block, False, "prefill", scale, None,
                        q=q, k=k, v=v)
    nb = nt
    mask = np.ones((Hq, nb, nb), dtype=np.uint8)
    ref = _check(w, lam, mask, f"jump d{d} b{block} lam{lam}")
    # the jump really happened: the last tile's rows end far above their first tile's max
    assert (ref["lse"][0, :, r0:] > 15).all()


@pytest.mark.parametrize("a", [0.0, 10.0, 1000.0])
def test_blasst_prefill_one_head_per_kv_head(a):
    """Causal BLASST prefill with one query head per KV head and several
    sequences (the shape of the BLASST page's Table 4 prefill, shrunk): the
    single-query-tile kernel."""
    B, H, N = 3, 1, 2048 + 96
    q, k, v = inputs.blasst_prefill_qkv(B, H, H, N, 128, "cpu", 4242)
    w = inputs.Workload("t4", B, H, H, N, 128, 128, True, "prefill", 1 / math.sqrt(128), None,
                        q=q, k=k, v=v)
    _check(w, inputs.lambda_for(a, N), None, f"table4-shape a={a}")


@pytest.mark.parametrize("hq,hkv,block,causal", [
    (4, 2, 128, True),     # two heads of one KV head per CTA
    (1, 1, 128, True),     # two consecutive query tiles per CTA, odd count
    (3, 1, 128, False),    # two consecutive query tiles, non-causal
    (2, 1, 64, True),      # one query tile per CTA
])
def test_reverse_visit_order(hq, hkv, block, causal):
    """Block-row reordering: every query tile visits its key tiles in
    descending order; decisions, O, LSE and tile status match the oracle's
    reversed visit.  Inputs: the first key of tile j scores 3 (j + 1) against
    every query and the rest score near 0, so the descending visit meets the
    largest score first and skips the earlier tiles (ln 0.1 > -3), while the
    ascending visit keeps every tile."""
    N = 5 * block + 21
    g = torch.Generator().manual_seed(21 + block)
    q = 0.1 * torch.randn(2, hq, N, 128, generator=g)
    q[..., 0] = 1.0
    k = 0.1 * torch.randn(2, hkv, N, 128, generator=g)
    for j in range(-(-N // block)):
        k[:, :, j * block, 0] = 3.0 * (j + 1)
    v = torch.randn(2, hkv, N, 128, generator=g)
    q, k, v = (x.to(torch.bfloat16) for x in (q, k, v))
    w = inputs.Workload("rev", 2, hq, hkv, N, 128, block, causal, "prefill", 1.0, None,
                        q=q, k=k, v=v)
    ref = _check(w, 0.1, None, f"reverse h{hq}/{hkv} b{block} c{causal}", reverse=True)
    assert (ref["status"] == 1).sum() > 0
    ref = _check(w, 0.1, None, f"ascending h{hq}/{hkv} b{block} c{causal}")
    assert (ref["status"] == 1).sum() == 0


@pytest.mark.parametrize("block", [64, 128])
def test_reverse_visit_order_with_masks(block):
    """Reverse order over per-head and shared block masks (CSR visit lists)."""
    rng = np.random.default_rng(block)
    N = 6 * block - 3
    nb = -(-N // block)
    q, k, v = inputs.blasst_prefill_qkv(1, 4, 2, N, 64, "cpu", 8)
    w = inputs.Workload("revm", 1, 4, 2, N, 64, block, True, "prefill", 0.125, None,
                        q=q, k=k, v=v)
    for heads in (1, 4):
        m = (rng.random((heads, nb, nb)) < 0.6).astype(np.uint8)
        m[:, np.arange(nb), np.arange(nb)] = 1
        _check(w, 0.02, m, f"reverse mask{heads}", reverse=True)


@pytest.mark.parametrize("hq,hkv,block,causal,masked", [
    (4, 2, 128, True, False),    # two heads of one KV head per CTA
    (1, 1, 128, True, False),    # two consecutive query tiles per CTA
    (2, 1, 128, False, False),
    (2, 1, 64, True, False),     # one query tile per CTA
    (4, 2, 128, True, True),     # per-head masks: one query tile per CTA
])
@pytest.mark.parametrize("reverse", [False, True])
def test_skip_v_loads(hq, hkv, block, causal, masked, reverse):
    """V tiles loaded only for executed tiles: the results are those of the
    oracle (which has no notion of loads) in either visit order."""
    N = 6 * block + 45
    q, k, v = inputs.blasst_prefill_qkv(1, hq, hkv, N, 128, "cpu", 77 + block)
    w = inputs.Workload("skipv", 1, hq, hkv, N, 128, block, causal, "prefill",
                        1 / math.sqrt(128), None, q=q, k=k, v=v)
    mask = None
    if masked:
        nb = -(-N // block)
        rng = np.random.default_rng(3)
        mask = (rng.random((hq, nb, nb)) < 0.7).astype(np.uint8)
        mask[:, np.arange(nb), np.arange(nb)] = 1
    ref = _check(w, 0.02, mask, f"skip_v h{hq}/{hkv} b{block} rev{reverse}", reverse=reverse,
                 skip_v=True)
    if not reverse:
        assert (ref["status"] == 1).sum() > 0


def test_skip_v_dense_and_full_size_sampled():
    """lambda = 0 with V skipping (every V tile is needed), and the full-size
    BLASST prefill with V skipping on sampled query tiles."""
    w = inputs.workload("blasst_prefill", shrink=True)
    _check(w, 0.0, None, "skip_v dense", skip_v=True)
    w = inputs.workload("blasst_prefill", device="cuda")
    lam = inputs.lambda_for(10.0, w.N)
    o, lse, st = _run_gpu(w, lam, None, skip_v=True)
    items = _sampled_items(w, 12, 9)
    ref = oracle.prefill(w.q.cpu(), w.k.cpu(), w.v.cpu(), w.block, w.scale, w.causal, lam,
                         items=items)
    o_c, lse_c, st_c = o.float().cpu().numpy(), lse.cpu().numpy(), st.cpu().numpy()
    for (b, h, i) in items:
        rows = slice(i * w.block, min(w.N, (i + 1) * w.block))
        compare_outputs(o_c[b, h, rows], ref["o"][b, h, rows], lse_c[b, h, rows],
                        ref["lse"][b, h, rows], f"skip_v item {(b, h, i)}")
        compare_status(st_c[b, h, i], ref["status"][b, h, i], ref["margin"][b, h, i])


@pytest.mark.parametrize("hq,hkv,block,causal,masked", [
    (4, 2, 128, True, False),    # two heads of one KV head per CTA
    (2, 2, 128, True, False),    # two consecutive query tiles per CTA
    (1, 1, 128, False, False),
    (2, 1, 64, True, False),     # one query tile per CTA
    (4, 2, 128, False, True),    # shared mask: two heads per CTA, CSR visit lists
    (4, 4, 64, True, True),      # per-head masks
])
@pytest.mark.parametrize("reverse", [False, True])
def test_varlen_key_padding(hq, hkv, block, causal, masked, reverse):
    """Per-sequence valid lengths (key padding): every kernel against the
    oracle's padded batch, lengths 0, partial tiles, tile multiples and full."""
    B, N = 5, 6 * block + 29
    lens = [N, 3 * block + 5, block, 0, 17]
    q, k, v = inputs.blasst_prefill_qkv(B, hq, hkv, N, 128, "cpu", 91 + block)
    ops = _ops()
    rp = ci = None
    mh = 1
    mask = None
    nb = -(-N // block)
    if masked:
        rng = np.random.default_rng(11)
        heads = 1 if hq != hkv else hq
        mask = (rng.random((heads, nb, nb)) < 0.6).astype(np.uint8)
        mask[:, np.arange(nb), np.arange(nb)] = 1
        m = torch.as_tensor(mask).cuda().contiguous()
        rp, ci, _ = ops.bsattn_build_index(m, block, block, causal)
        mh = heads
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    st = torch.zeros(B, hq, nb, nb, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lam = 0.02
    o, lse = ops.bsattn_fwd_prefill(q.cuda(), k.cuda(), v.cuda(), block, 1 / math.sqrt(128),
                                    causal, lam, rp, ci, mh, tile_status=st, status=status,
                                    reverse=reverse, seq_lens=sl)
    torch.cuda.synchronize()
    assert status.item() == 0, ops.bsattn_status_string(status.item())
    ref = oracle.prefill(q, k, v, block, 1 / math.sqrt(128), causal, lam, mask=mask,
                         reverse=reverse, seq_lens=lens)
    compare_outputs(o, ref["o"], lse, ref["lse"], f"varlen h{hq}/{hkv} b{block} rev{reverse}")
    compare_status(st, ref["status"], ref["margin"], "varlen")
    for b, L in enumerate(lens):     # padding rows: exactly zero and -inf
        assert (o[b, :, L:].float() == 0).all()
        assert torch.isneginf(lse[b, :, L:]).all()


@pytest.mark.parametrize("masked", [None, "shared", "per_head"])
@pytest.mark.parametrize("chunk", [1, 2])
def test_host_pipeline_equals_device_path(masked, chunk):
    """bsattn_fwd_prefill_host (host buffers, per-chunk copies overlapped with
    the kernels) gives exactly the output of the device path."""
    ops = _ops()
    B, Hq, Hkv, N, block = 2, 8, 2, 5 * 128 + 37, 128
    q, k, v = inputs.blasst_prefill_qkv(B, Hq, Hkv, N, 128, "cpu", 44)
    lam = 0.02
    rp = ci = order = None
    mh = 1
    if masked:
        nb = -(-N // block)
        heads = 1 if masked == "shared" else Hq
        rng = np.random.default_rng(6)
        m = (rng.random((heads, nb, nb)) < 0.6).astype(np.uint8)
        m[:, np.arange(nb), np.arange(nb)] = 1
        rp, ci, _, order = ops.bsattn_build_index(torch.as_tensor(m).cuda(), block, block, True,
                                                  with_order=True)
        mh = heads
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    ref, _ = ops.bsattn_fwd_prefill(qd, kd, vd, block, None, True, lam, rp, ci, mh,
                                    row_order=order, want_lse=False)
    hq, hk, hv = q.pin_memory(), k.pin_memory(), v.pin_memory()
    ho = torch.empty_like(q).pin_memory()
    sq, sk, sv, so = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd), \
        torch.empty_like(qd)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.bsattn_fwd_prefill_host(hq, hk, hv, ho, sq, sk, sv, so, block, None, True, lam, rp, ci,
                                mh, row_order=order, kv_heads_per_chunk=chunk, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(ho, ref.cpu())


def test_long_sequence_sampled():
    """A 131,149-token causal prefill (1,025 query tiles, 1,050,625 tile-status
    entries per head) with the skip on: sampled query tiles, including the
    last and ragged one, against the oracle."""
    B, Hq, Hkv, N = 1, 2, 1, 131072 + 77
    q, k, v = inputs.blasst_prefill_qkv(B, Hq, Hkv, N, 128, "cuda", 321)
    w = inputs.Workload("long", B, Hq, Hkv, N, 128, 128, True, "prefill", 1 / math.sqrt(128),
                        None, q=q, k=k, v=v)
    lam = inputs.lambda_for(10.0, N)
    o, lse, st = _run_gpu(w, lam, None)
    items = [(0, 0, 0), (0, 1, 513), (0, 0, 1024), (0, 1, 1024), (0, 0, 700)]
    ref = oracle.prefill(q.cpu(), k.cpu(), v.cpu(), 128, w.scale, True, lam, items=items)
    o_c, lse_c, st_c = o.float().cpu().numpy(), lse.cpu().numpy(), st.cpu().numpy()
    for (b, h, i) in items:
        rows = slice(i * 128, min(N, (i + 1) * 128))
        compare_outputs(o_c[b, h, rows], ref["o"][b, h, rows], lse_c[b, h, rows],
                        ref["lse"][b, h, rows], f"long item {(b, h, i)}")
        compare_status(st_c[b, h, i], ref["status"][b, h, i], ref["margin"][b, h, i])


def test_short_sequence_single_partial_tile():
    q, k, v = inputs.normal_qkv(1, 2, 2, 50, 128, "cpu", 3)
    w = inputs.Workload("short", 1, 2, 2, 50, 128, 128, True, "prefill", 1 / math.sqrt(128), None,
                        q=q, k=k, v=v)
    _check(w, 0.5, None, "short")


def test_closed_form_skip_on_gpu():
    """The two-tile closed form of the oracle pins, on the GPU (block 64, d 64)."""
    N, d = 128, 64
    qn = np.zeros((N, d)); qn[:, 0] = 1.0
    kn = np.zeros((N, d)); kn[0, 0] = 10.0; kn[64:, 0] = 2.0
    vn = np.round(np.random.default_rng(0).standard_normal((N, d)) * 8) / 8
    t = lambda x: torch.tensor(x, dtype=torch.float32).to(torch.bfloat16)[None, None].contiguous()
    w = inputs.Workload("cf", 1, 1, 1, N, d, 64, False, "prefill", 1.0, None, q=t(qn), k=t(kn), v=t(vn))
    o, lse, st = _run_gpu(w, math.exp(-5))
    assert (st[0, 0, :, 1] == 1).all() and (st[0, 0, :, 0] == 2).all()
    expect = (math.exp(10) * vn[0] + vn[1:64].sum(0)) / (math.exp(10) + 63)
    assert np.abs(o[0, 0].float().cpu().numpy() - expect[None]).max() < 2e-2


def _sampled_items(w, n_items, seed):
    rng = np.random.default_rng(seed)
    items = set()
    # always include the first and the last query tile of some heads
    for h in rng.choice(w.Hq, size=min(2, w.Hq), replace=False):
        items.add((0, int(h), 0))
        items.add((0, int(h), w.nq - 1))
    while len(items) < n_items:
        items.add((int(rng.integers(w.B)), int(rng.integers(w.Hq)), int(rng.integers(w.nq))))
    return sorted(items)


def _check_sampled(w, lam, mask, n_items, what):
    """Full-size workload in the launch configuration the benchmark times,
    compared on sampled query tiles that the oracle computes one by one."""
    o, lse, st = _run_gpu(w, lam, mask)
    items = _sampled_items(w, n_items, 5)
    ref = oracle.prefill(w.q.cpu(), w.k.cpu(), w.v.cpu(), w.block, w.scale, w.causal, lam,
                         mask=mask, items=items)
    o_c, lse_c, st_c = o.float().cpu().numpy(), lse.cpu().numpy(), st.cpu().numpy()
    for (b, h, i) in items:
        rows = slice(i * w.block, min(w.N, (i + 1) * w.block))
        compare_outputs(o_c[b, h, rows], ref["o"][b, h, rows], lse_c[b, h, rows],
                        ref["lse"][b, h, rows], f"{what} item {(b, h, i)}")
        compare_status(st_c[b, h, i], ref["status"][b, h, i], ref["margin"][b, h, i],
                       f"{what} item {(b, h, i)}")


def test_videodit_full_size_sampled():
    w = inputs.workload("videodit", device="cuda")
    _check_sampled(w, 0.0, w.mask.numpy(), 24, "videodit")


@pytest.mark.parametrize("a", [0.0, 10.0])
def test_blasst_prefill_full_size_sampled(a):
    w = inputs.workload("blasst_prefill", device="cuda")
    _check_sampled(w, inputs.lambda_for(a, w.N), None, 24, f"blasst a={a}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("lam", [0.0, 3e-3])
@pytest.mark.parametrize("per_head", [False, True])
def test_masks_rows_of_their_own(d, causal, lam, per_head):
    """Masks whose rows no two query tiles share (one query head per KV head,
    or one mask per head) with 128-token tiles: an odd number of query tiles,
    rows of very different lengths, empty rows and a ragged tail."""
    rng = np.random.default_rng(d + 2 * causal + (lam > 0) + 4 * per_head)
    B, Hq, Hkv, N = 1, 3, 3 if not per_head else 1, 5 * 128 - 17
    nb = -(-N // 128)
    hm = Hq if per_head else 1
    m = (rng.random((hm, nb, nb)) < 0.5).astype(np.uint8)
    m[:, np.arange(nb), np.arange(nb)] = 1
    m[:, 0, :] = 1                                 # a long row next to short ones
    m[:, 3, :] = 0                                 # an empty row
    q, k, v = inputs.blasst_prefill_qkv(B, Hq, Hkv, N, d, "cpu", 91 + d)
    w = inputs.Workload("own", B, Hq, Hkv, N, d, 128, causal, "prefill", 1 / math.sqrt(d), None,
                        q=q, k=k, v=v)
    assert (B * Hq * nb) % 2 == 1
    o, lse, st = _run_gpu(w, lam, m)
    ref = oracle.prefill(q, k, v, 128, w.scale, causal, lam, mask=m)
    compare_outputs(o, ref["o"], lse, ref["lse"], f"d{d} causal={causal} lam={lam}")
    compare_status(st, ref["status"], ref["margin"], f"d{d} causal={causal} lam={lam}")
    rows = slice(3 * 128, 4 * 128)
    assert (o[:, :, rows].float() == 0).all()
    assert torch.isneginf(lse[:, :, rows]).all()


@pytest.mark.parametrize("lam", [1.0, 1e-30])
@pytest.mark.parametrize("hq,hkv,block,masked", [(4, 2, 128, False), (2, 2, 64, False),
                                                 (3, 3, 128, True)])
def test_lambda_at_the_ends_of_its_range(lam, hq, hkv, block, masked):
    """lambda = 1 (the largest allowed: a tile is skipped unless some row
    reaches the running max) and lambda = 1e-30 (effectively no skipping), on
    the two-tile kernel, 64-token tiles and a shared mask with one query head
    per KV head."""
    N = 5 * block + 23
    nb = -(-N // block)
    q, k, v = inputs.blasst_prefill_qkv(1, hq, hkv, N, 128, "cpu", 61 + block)
    w = inputs.Workload("ends", 1, hq, hkv, N, 128, block, True, "prefill", 1 / math.sqrt(128),
                        None, q=q, k=k, v=v)
    mask = None
    if masked:
        rng = np.random.default_rng(62)
        mask = (rng.random((1, nb, nb)) < 0.7).astype(np.uint8)
        mask[:, np.arange(nb), np.arange(nb)] = 1
    ref = _check(w, lam, mask, f"lambda {lam} h{hq}/{hkv} b{block}")
    if lam == 1.0:
        assert (ref["status"] == 1).sum() > 0
