"""Independent fp64 references used to pin the oracle (numpy only).

``dense_attention`` is the textbook softmax(scale * q k^T + M) v ("Attention
的七十二变", section 1; masked_fill with -inf for excluded positions, section
2.2), written with numpy's matmul, max, exp and sum.  It is not the oracle's
algorithm (no tiles, no running max, no skip test), so agreement on the
lambda = 0 cases pins the oracle's scores, masking, scale, GQA indexing and
normalisation.
"""
import numpy as np


def bf16_to_f64(t):
    import torch
    b = t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def dense_attention(q64, k64, v64, scale, allowed=None):
    """q [n, d], k/v [L, d]; allowed bool [n, L].  Rows with no allowed key
    give zeros and -inf."""
    s = (q64 @ k64.T) * scale
    if allowed is not None:
        s = np.where(allowed, s, -np.inf)
    mu = s.max(axis=1, keepdims=True)
    ok = np.isfinite(mu[:, 0])
    mu = np.where(np.isfinite(mu), mu, 0.0)
    p = np.exp(s - mu)
    z = p.sum(axis=1, keepdims=True)
    out = np.zeros((q64.shape[0], v64.shape[1]))
    out[ok] = (p[ok] @ v64) / z[ok]
    lse = np.full(q64.shape[0], -np.inf)
    lse[ok] = mu[ok, 0] + np.log(z[ok, 0])
    return out, lse


def element_mask(block_mask, block, N, causal):
    """Expand a [nq, nk] block mask to a token-level [N, N] boolean mask,
    adding the causal rule key <= query."""
    bm = np.asarray(block_mask, dtype=bool)
    e = np.repeat(np.repeat(bm, block, axis=0), block, axis=1)[:N, :N]
    if causal:
        e &= np.tril(np.ones((N, N), dtype=bool))
    return e
