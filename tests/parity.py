"""Comparison helpers for the GPU parity tests (CUDA library vs fp64 oracle).

Tolerances are the ones the task states for this path: bf16 inputs -> max-abs
2e-2 and mean-abs 2e-3 on O, 1e-2 on the LSE; fp32 inputs -> 1e-4 max-abs.
"""
import numpy as np
import torch

BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
LSE_ABS = 1e-2
F32_MAX_ABS = 1e-4


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def check(out, lse, ref_out, ref_lse, *, max_abs, mean_abs=None, lse_abs=LSE_ABS, what=""):
    """Element-wise comparison; returns a dict of error statistics."""
    out = np.asarray(out, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    assert out.shape == ref_out.shape, (out.shape, ref_out.shape)
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    assert np.isfinite(lse).all(), f"{what}: non-finite lse"
    err = np.abs(out - ref_out)
    lerr = np.abs(lse - ref_lse)
    rel = err.max() / max(np.abs(ref_out).max(), 1e-30)
    stats = dict(max_abs=float(err.max()), mean_abs=float(err.mean()),
                 lse_max_abs=float(lerr.max()), rel_to_max=float(rel))
    assert err.max() <= max_abs, f"{what}: max-abs {err.max():.3e} > {max_abs} {stats}"
    if mean_abs is not None:
        assert err.mean() <= mean_abs, f"{what}: mean-abs {err.mean():.3e} > {mean_abs} {stats}"
    assert lerr.max() <= lse_abs, f"{what}: lse max-abs {lerr.max():.3e} > {lse_abs} {stats}"
    return stats


def gather_rows(out, lse, rb, rq, rh):
    """GPU out [B,L,Hq,D] / lse [B,Hq,L] at rows (b, q, h) -> numpy."""
    dev = out.device
    b = torch.as_tensor(rb, dtype=torch.long, device=dev)
    q = torch.as_tensor(rq, dtype=torch.long, device=dev)
    h = torch.as_tensor(rh, dtype=torch.long, device=dev)
    return to_np(out[b, q, h]), to_np(lse[b, h, q])
