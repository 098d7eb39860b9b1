"""Tolerance check shared by the GPU parity tests.

The bar (from the hot path's statement of accuracy): against the float64
oracle on the same bf16 inputs,
  * O: max |O_gpu - O_ref| <= 1e-2 and ||O_gpu - O_ref||_2 / ||O_ref||_2 <= 5e-3
    over the checked set;
  * LSE: every -inf of the oracle (row with no visible key) is -inf on the GPU
    and vice versa; elsewhere max |LSE_gpu - LSE_ref| <= 1e-3;
  * no NaN anywhere.
"""
from __future__ import annotations

import numpy as np

O_MAX_ABS = 1e-2
O_REL_RMS = 5e-3
LSE_MAX_ABS = 1e-3


def to_f64(x) -> np.ndarray:
    import torch
    if isinstance(x, torch.Tensor):
        return x.detach().float().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def check(o_gpu, o_ref, lse_gpu=None, lse_ref=None, what=""):
    """Raise AssertionError with statistics when the GPU result misses the bar."""
    og = to_f64(o_gpu).reshape(-1)
    orf = to_f64(o_ref).reshape(-1)
    assert og.shape == orf.shape, f"{what}: shape {og.shape} vs {orf.shape}"
    assert not np.isnan(og).any(), f"{what}: NaN in O"
    assert np.isfinite(og).all(), f"{what}: inf in O"
    diff = og - orf
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    ref_norm = float(np.linalg.norm(orf))
    rel_rms = float(np.linalg.norm(diff) / ref_norm) if ref_norm > 0 else float(np.linalg.norm(diff))
    stats = {"o_max_abs": max_abs, "o_rel_rms": rel_rms}
    if lse_gpu is not None:
        lg = to_f64(lse_gpu).reshape(-1)
        lr = to_f64(lse_ref).reshape(-1)
        assert not np.isnan(lg).any(), f"{what}: NaN in LSE"
        ninf_ref = np.isneginf(lr)
        ninf_gpu = np.isneginf(lg)
        mism = int((ninf_ref != ninf_gpu).sum())
        assert mism == 0, f"{what}: {mism} rows disagree on being empty (-inf LSE)"
        fin = ~ninf_ref
        lse_err = float(np.abs(lg[fin] - lr[fin]).max()) if fin.any() else 0.0
        stats["lse_max_abs"] = lse_err
        stats["empty_rows"] = int(ninf_ref.sum())
        assert lse_err <= LSE_MAX_ABS, f"{what}: LSE max abs {lse_err:.3e} > {LSE_MAX_ABS} {stats}"
    assert max_abs <= O_MAX_ABS, f"{what}: O max abs {max_abs:.3e} > {O_MAX_ABS} {stats}"
    assert rel_rms <= O_REL_RMS, f"{what}: O rel RMS {rel_rms:.3e} > {O_REL_RMS} {stats}"
    return stats
