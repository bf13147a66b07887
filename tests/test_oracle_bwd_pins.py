"""Pins for the oracle's backward pass (sparsity-aware training, BLASST page
section 3.3: the forward applies the skip and the blocks it skipped receive no
gradient).  The gradient is tied to things other than itself: torch's fp64
autograd of the textbook softmax attention where the executed set is plain
(dense, a static block mask, or the executed tiles as an element mask),
central differences of the forward oracle itself with skips present, closed
forms (constant keys give dQ = 0; zero queries give uniform attention), the
zero gradient of never-executed keys, the GQA group sum, and key padding.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_bsattn_b200 import inputs
from tests._refs import bf16_to_f64, element_mask

H = 2.0 ** -7   # grid step: multiples of H in (-1, 1) are exact in bf16, and stay so after +-H


def _bf16(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


def _dout(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _autograd(q, k, v, dout, scale, allowed):
    """Gradients of sum(dout * softmax(scale q k^T masked) v) by torch fp64
    autograd; allowed bool [B, Hq, N, N]; K/V repeated over the GQA group."""
    Q = torch.tensor(bf16_to_f64(q), requires_grad=True)
    K = torch.tensor(bf16_to_f64(k), requires_grad=True)
    V = torch.tensor(bf16_to_f64(v), requires_grad=True)
    g = Q.shape[1] // K.shape[1]
    s = scale * Q @ K.repeat_interleave(g, 1).transpose(-1, -2)
    al = torch.from_numpy(np.array(allowed, dtype=bool))
    s = s.masked_fill(~al, float("-inf"))
    p = torch.softmax(s, -1).nan_to_num(0.0)          # rows without keys: no weight
    o = p @ V.repeat_interleave(g, 1)
    (o * torch.as_tensor(dout)).sum().backward()
    return Q.grad.numpy(), K.grad.numpy(), V.grad.numpy()


def _close(a, b, tol=1e-12):
    assert np.abs(a - b).max() <= tol * max(1.0, np.abs(b).max()), np.abs(a - b).max()


# ------------------------------------------------- library routine on plain executed sets
@pytest.mark.parametrize("B,Hq,Hkv,N,d,block,causal", [
    (1, 2, 2, 160, 32, 64, False),
    (2, 4, 2, 200, 64, 64, True),      # GQA, ragged tail, causal
    (1, 3, 1, 130, 64, 128, True),     # MQA, odd group, ragged tail
])
def test_bwd_dense_equals_autograd(B, Hq, Hkv, N, d, block, causal):
    """lambda = 0 and no mask: the plain softmax attention gradient."""
    q, k, v = inputs.normal_qkv(B, Hq, Hkv, N, d, "cpu", 11)
    scale = 1.0 / math.sqrt(d)
    f = oracle.prefill(q, k, v, block, scale, causal, 0.0)
    do = _dout(q.shape, 12)
    r = oracle.prefill_bwd(q, k, v, do, block, scale, causal, f["status"])
    nb = -(-N // block)
    allowed = np.broadcast_to(element_mask(np.ones((nb, nb)), block, N, causal), (B, Hq, N, N))
    dq, dk, dv = _autograd(q, k, v, do, scale, allowed)
    _close(r["dq"], dq)
    _close(r["dk"], dk)
    _close(r["dv"], dv)


def test_bwd_static_mask_equals_autograd_with_element_mask():
    """A per-head static block mask (causal, GQA): gradients of the
    element-masked softmax; masked-out blocks get nothing."""
    B, Hq, Hkv, N, d, block = 1, 4, 2, 256, 32, 64
    q, k, v = inputs.normal_qkv(B, Hq, Hkv, N, d, "cpu", 13)
    nb = N // block
    rng = np.random.default_rng(14)
    mask = (rng.random((Hq, nb, nb)) < 0.5).astype(np.uint8)
    mask[:, np.arange(nb), np.arange(nb)] = 1
    scale = 0.2
    f = oracle.prefill(q, k, v, block, scale, True, 0.0, mask=mask)
    do = _dout(q.shape, 15)
    r = oracle.prefill_bwd(q, k, v, do, block, scale, True, f["status"])
    allowed = np.stack([element_mask(mask[h], block, N, True) for h in range(Hq)])[None]
    dq, dk, dv = _autograd(q, k, v, do, scale, allowed)
    _close(r["dq"], dq)
    _close(r["dk"], dk)
    _close(r["dv"], dv)


def test_bwd_blasst_equals_autograd_over_executed_tiles():
    """With skips (the sink recipe, a = 10): the gradient is that of the
    softmax over the executed tiles' keys, i.e. autograd with the forward's
    executed tiles as the element mask."""
    B, Hq, Hkv, N, d, block = 1, 4, 2, 640, 64, 64
    q, k, v = inputs.blasst_prefill_qkv(B, Hq, Hkv, N, d, "cpu", 1237)
    scale = 1.0 / math.sqrt(d)
    lam = 10.0 / N
    f = oracle.prefill(q, k, v, block, scale, True, lam)
    assert (f["status"] == 1).sum() > 0 and (f["status"] == 2).sum() > 0
    do = _dout(q.shape, 16)
    r = oracle.prefill_bwd(q, k, v, do, block, scale, True, f["status"])
    ex = f["status"] == 2
    allowed = np.stack([element_mask(ex[0, h], block, N, True) for h in range(Hq)])[None]
    dq, dk, dv = _autograd(q, k, v, do, scale, allowed)
    _close(r["dq"], dq)
    _close(r["dk"], dk)
    _close(r["dv"], dv)


# ------------------------------------------------------------- central differences
def _grid_case(seed, B=1, Hq=2, Hkv=1, N=192, d=16):
    """Grid inputs (multiples of H in (-1, 1)) with a shared direction u:
    queries lean on u; keys of tiles 0 and 2 are u plus noise, tile 1 noise
    only, so with scale 2 and ln(lambda) = -2 every query tile keeps tiles 0
    and 2 and skips tile 1, all margins above 1."""
    rng = np.random.default_rng(seed)

    def grid(shape, lim):
        return rng.integers(-int(lim / H), int(lim / H) + 1, size=shape) * H

    u = rng.choice([-0.75, 0.75], size=(B, Hkv, 1, d))
    q = 0.375 * np.repeat(u, Hq // Hkv, axis=1) + grid((B, Hq, N, d), 0.25)
    k = grid((B, Hkv, N, d), 0.5)
    k[:, :, :64] = u + grid((B, Hkv, 64, d), 0.125)
    k[:, :, 128:] = u + grid((B, Hkv, 64, d), 0.125)
    v = grid((B, Hkv, N, d), 0.875)
    return q, k, v


@pytest.mark.parametrize("which", ["q", "k", "v"])
def test_bwd_central_differences_with_skips(which):
    """(L(x + hU) - L(x - hU)) / 2 = <grad, U> for L = sum(dO * O) of the
    forward oracle, in a case where tile 1 is skipped and the perturbation
    flips no decision."""
    scale, lam, block = 2.0, math.exp(-2.0), 64
    q, k, v = _grid_case(3)
    do = _dout(q.shape, 17)
    f = oracle.prefill(_bf16(q), _bf16(k), _bf16(v), block, scale, False, lam)
    st = f["status"]
    assert (st == 1).sum() == 6 and (st == 2).sum() == 12
    assert np.abs(f["margin"][st > 0][np.isfinite(f["margin"][st > 0])]).min() > 1.0
    g = oracle.prefill_bwd(_bf16(q), _bf16(k), _bf16(v), do, block, scale, False, st)
    g = {"q": g["dq"], "k": g["dk"], "v": g["dv"]}[which]
    x = {"q": q, "k": k, "v": v}
    U = np.random.default_rng(18).choice([-1.0, 0.0, 0.0, 0.0, 1.0], size=x[which].shape) * H
    out = []
    for sgn in (1.0, -1.0):
        xs = dict(x)
        xs[which] = x[which] + sgn * U
        assert np.array_equal(bf16_to_f64(_bf16(xs[which])), xs[which])   # exact in bf16
        r = oracle.prefill(_bf16(xs["q"]), _bf16(xs["k"]), _bf16(xs["v"]), block, scale, False,
                           lam)
        assert np.array_equal(r["status"], st)
        out.append((r["o"] * do).sum())
    fd = (out[0] - out[1]) / 2.0
    an = (g * U).sum()
    assert abs(fd - an) <= 1e-4 * np.linalg.norm(g) * np.linalg.norm(U), (fd, an)


# ------------------------------------------------------------- invariants, closed forms
def test_bwd_never_executed_keys_get_no_gradient():
    """Keys of tiles that no query tile executed: dK = dV = 0 exactly, and the
    other gradients do not depend on their values."""
    scale, lam, block = 2.0, math.exp(-2.0), 64
    q, k, v = _grid_case(5)
    do = _dout(q.shape, 19)
    f = oracle.prefill(_bf16(q), _bf16(k), _bf16(v), block, scale, False, lam)
    st = f["status"]
    assert (st[:, :, :, 1] == 1).all()                    # tile 1 skipped everywhere
    r = oracle.prefill_bwd(_bf16(q), _bf16(k), _bf16(v), do, block, scale, False, st)
    assert (r["dk"][:, :, 64:128] == 0).all() and (r["dv"][:, :, 64:128] == 0).all()
    assert np.abs(r["dk"][:, :, :64]).max() > 0 and np.abs(r["dv"][:, :, 128:]).max() > 0
    k2, v2 = k.copy(), v.copy()
    k2[:, :, 64:128] = -k2[:, :, 64:128]
    v2[:, :, 64:128] = 0.5
    r2 = oracle.prefill_bwd(_bf16(q), _bf16(k2), _bf16(v2), do, block, scale, False, st)
    for key in ("dq", "dk", "dv"):
        assert np.array_equal(r2[key], r[key])


def test_bwd_constant_keys_give_zero_dq():
    """All keys equal: dS sums to zero along every row (the softmax Jacobian
    kills constants), so dQ = scale * sum_c dS_rc k = 0."""
    B, Hq, Hkv, N, d, block = 1, 2, 1, 192, 32, 64
    q, _, v = inputs.normal_qkv(B, Hq, Hkv, N, d, "cpu", 21)
    kc = torch.randn(d, generator=torch.Generator().manual_seed(22)).to(torch.bfloat16)
    k = kc.expand(B, Hkv, N, d).contiguous()
    f = oracle.prefill(q, k, v, block, 0.3, True, 0.0)
    r = oracle.prefill_bwd(q, k, v, _dout(q.shape, 23), block, 0.3, True, f["status"])
    assert np.abs(r["dq"]).max() < 1e-12
    assert np.abs(r["dv"]).max() > 0.1


def test_bwd_zero_queries_uniform_attention():
    """q = 0: every allowed key gets weight 1/n_r, so dV_c = sum over rows r
    that see c of dO_r / n_r (n_r = r + 1 under the causal rule), and dK = 0."""
    B, Hq, Hkv, N, d, block = 1, 2, 1, 150, 16, 64
    _, k, v = inputs.normal_qkv(B, Hq, Hkv, N, d, "cpu", 24)
    q = torch.zeros(B, Hq, N, d, dtype=torch.bfloat16)
    f = oracle.prefill(q, k, v, block, 1.0, True, 0.0)
    do = _dout(q.shape, 25)
    r = oracle.prefill_bwd(q, k, v, do, block, 1.0, True, f["status"])
    want = np.zeros((N, d))
    for h in range(Hq):
        for t in range(N):
            want[: t + 1] += do[0, h, t] / (t + 1)
    _close(r["dv"][0, 0], want)
    assert np.abs(r["dk"]).max() < 1e-12


def test_bwd_gqa_equals_group_sum_of_mha():
    """A KV head's dK and dV are the sums of the per-head gradients of the
    same problem with K and V repeated for every query head."""
    B, Hq, Hkv, N, d, block = 1, 4, 2, 200, 32, 64
    q, k, v = inputs.normal_qkv(B, Hq, Hkv, N, d, "cpu", 26)
    g = Hq // Hkv
    lam = 0.05
    do = _dout(q.shape, 27)
    f = oracle.prefill(q, k, v, block, 0.4, True, lam)
    r = oracle.prefill_bwd(q, k, v, do, block, 0.4, True, f["status"])
    kr, vr = k.repeat_interleave(g, 1), v.repeat_interleave(g, 1)
    fm = oracle.prefill(q, kr, vr, block, 0.4, True, lam)
    assert np.array_equal(fm["status"], f["status"])
    rm = oracle.prefill_bwd(q, kr, vr, do, block, 0.4, True, fm["status"])
    _close(r["dq"], rm["dq"])
    _close(r["dk"], rm["dk"].reshape(B, Hkv, g, N, d).sum(2))
    _close(r["dv"], rm["dv"].reshape(B, Hkv, g, N, d).sum(2))


@pytest.mark.parametrize("causal", [True, False])
def test_bwd_varlen_equals_each_sequence_alone(causal):
    """Key padding: a padded batch's gradients equal each sequence's own;
    padding query rows, keys and values get zero gradient (without the causal
    rule the padding keys of a partly valid tile are the ones at stake)."""
    B, Hq, Hkv, N, d, block = 3, 2, 1, 192, 32, 64
    q, k, v = inputs.normal_qkv(B, Hq, Hkv, N, d, "cpu", 28)
    lens = [192, 130, 64]
    lam = 0.02
    do = _dout(q.shape, 29)
    f = oracle.prefill(q, k, v, block, 0.3, causal, lam, seq_lens=lens)
    r = oracle.prefill_bwd(q, k, v, do, block, 0.3, causal, f["status"], seq_lens=lens)
    for b, L in enumerate(lens):
        fs = oracle.prefill(q[b:b + 1, :, :L], k[b:b + 1, :, :L], v[b:b + 1, :, :L], block, 0.3,
                            causal, lam)
        rs = oracle.prefill_bwd(q[b:b + 1, :, :L], k[b:b + 1, :, :L], v[b:b + 1, :, :L],
                                do[b:b + 1, :, :L], block, 0.3, causal, fs["status"])
        for key in ("dq", "dk", "dv"):
            _close(r[key][b:b + 1, :, :L], rs[key])
            assert (r[key][b, :, L:] == 0).all()
