"""Comparison helpers shared by the GPU parity tests and the smoke check.

Bars (block-sparse attention with bf16 inputs and fp32 accumulation against
the fp64 oracle): max-abs <= 2e-2 and mean-abs <= 2e-3 on O; LSE within 1e-2;
tile status identical, except that a visited tile whose skip margin (tile
max minus running max minus ln(lambda), natural-log units) lies within 1e-3
of zero may go either way.
"""
import numpy as np
import torch

O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-2
MARGIN_TIE = 1e-3


def compare_outputs(o_gpu, ref_o, lse_gpu=None, ref_lse=None, what=""):
    o = o_gpu.float().cpu().numpy() if isinstance(o_gpu, torch.Tensor) else o_gpu
    err = np.abs(o - ref_o)
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    assert err.max() <= O_MAX_ABS, f"{what}: max-abs {err.max():.3e}"
    assert err.mean() <= O_MEAN_ABS, f"{what}: mean-abs {err.mean():.3e}"
    if lse_gpu is not None:
        lse = lse_gpu.float().cpu().numpy() if isinstance(lse_gpu, torch.Tensor) else lse_gpu
        both_inf = np.isneginf(lse) & np.isneginf(ref_lse)
        with np.errstate(invalid="ignore"):
            d = np.where(both_inf, 0.0, np.abs(lse - ref_lse))
        assert np.nanmax(d) <= LSE_MAX_ABS, f"{what}: lse max-abs {np.nanmax(d):.3e}"
    return float(err.max()), float(err.mean())


def compare_status(st_gpu, ref_status, ref_margin, what=""):
    st = st_gpu.cpu().numpy() if isinstance(st_gpu, torch.Tensor) else st_gpu
    st = st.astype(np.int32)
    rs = ref_status.astype(np.int32)
    assert ((st > 0) == (rs > 0)).all(), f"{what}: visited sets differ"
    differ = st != rs
    near = np.abs(ref_margin) < MARGIN_TIE
    bad = differ & ~near
    assert not bad.any(), f"{what}: {int(bad.sum())} executed-tile decisions differ " \
                          f"(of {int((rs > 0).sum())} visited)"
    return int(differ.sum())
