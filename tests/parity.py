"""Tolerance check shared by the GPU parity tests.

The bar (from the hot path's statement of accuracy): against the float64
oracle on the same bf16 inputs,
  * O: max |O_gpu - O_ref| <= 1e-2 and ||O_gpu - O_ref||_2 / ||O_ref||_2 <= 5e-3
    over the checked set;
  * LSE: every -inf of the oracle (row with no visible key) is -inf on the GPU
    and vice versa; elsewhere max |LSE_gpu - LSE_ref| <= 1e-3;
  * no NaN anywhere.

Gradients of the backward pass (dQ, dK, dV) are checked with
  * ||G_gpu - G_ref||_2 / ||G_ref||_2 <= 5e-3 (the forward's relative bar) and
  * max |G_gpu - G_ref| <= 2e-2 * max(1, max |G_ref|).
The scale-relative max bound follows from the arithmetic: the kernels round P
and dS to bf16 for the tensor cores and each gradient to bf16 on output, so
the error grows with the gradient's magnitude (gradients of keys seen by many
rows reach several units).  A float32 simulation of exactly those roundings
gives rel-RMS 2.3e-3 to 2.5e-3 and max |error| <= 4.6e-3 * max |G_ref| on
seeded N(0,1) inputs (d = 64 and 128, causal and not, S up to 1024).
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


GRAD_REL_RMS = 5e-3
GRAD_MAX_ABS_REL = 2e-2


def check_grad(g_gpu, g_ref, what=""):
    """Raise AssertionError when a gradient misses the bar stated above."""
    gg = to_f64(g_gpu).reshape(-1)
    gr = to_f64(g_ref).reshape(-1)
    assert gg.shape == gr.shape, f"{what}: shape {gg.shape} vs {gr.shape}"
    assert np.isfinite(gg).all(), f"{what}: non-finite gradient"
    diff = gg - gr
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    ref_max = float(np.abs(gr).max()) if gr.size else 0.0
    ref_norm = float(np.linalg.norm(gr))
    rel_rms = float(np.linalg.norm(diff) / ref_norm) if ref_norm > 0 else float(np.linalg.norm(diff))
    stats = {"max_abs": max_abs, "ref_max": ref_max, "rel_rms": rel_rms}
    assert max_abs <= GRAD_MAX_ABS_REL * max(1.0, ref_max), f"{what}: max abs {stats}"
    if ref_norm > 0:
        assert rel_rms <= GRAD_REL_RMS, f"{what}: rel RMS {stats}"
    else:
        assert max_abs == 0.0, f"{what}: expected exact zeros {stats}"
    return stats
