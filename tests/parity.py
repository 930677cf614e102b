"""Shared comparison rule for GPU-vs-oracle parity tests.

Bar (from the workload statement): bf16/fp32 outputs max-abs <= 2e-2 and
mean-abs <= 2e-3 against the float64 oracle; LSE within 1e-3 relative, with the
relative error floored at |lse| = 1 (LSE can be ~0, e.g. causal row 0).
"""
import numpy as np
import torch

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
LSE_REL = 1e-3


def to_np(t):
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


def check(out, ref_out, lse, ref_lse, what=""):
    out, ref_out, lse, ref_lse = to_np(out), to_np(ref_out), to_np(lse), to_np(ref_lse)
    assert out.shape == ref_out.shape, (what, out.shape, ref_out.shape)
    assert np.all(np.isfinite(out)), f"{what}: non-finite output"
    err = np.abs(out - ref_out)
    max_abs, mean_abs = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    assert max_abs <= MAX_ABS, f"{what}: max-abs {max_abs:.3e} > {MAX_ABS}"
    assert mean_abs <= MEAN_ABS, f"{what}: mean-abs {mean_abs:.3e} > {MEAN_ABS}"
    both_inf = np.isneginf(lse) & np.isneginf(ref_lse)
    assert np.array_equal(np.isneginf(lse), np.isneginf(ref_lse)), f"{what}: -inf LSE pattern differs"
    fin = ~both_inf
    lerr = np.abs(lse[fin] - ref_lse[fin]) / np.maximum(1.0, np.abs(ref_lse[fin]))
    lmax = float(lerr.max()) if lerr.size else 0.0
    assert lmax <= LSE_REL, f"{what}: lse rel err {lmax:.3e} > {LSE_REL}"
    return dict(max_abs=max_abs, mean_abs=mean_abs, lse_rel=lmax)
