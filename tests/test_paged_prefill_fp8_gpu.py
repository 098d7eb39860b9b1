"""GPU parity of attn_fwd_paged_fp8 (packed queries appended to an E4M3 paged
cache) against the oracles.

"Attention Kernel", sections "Paged 与 ragged KV" and "正确性契约": the cache
holds E4M3 codes with one scale per (page, KV head), element = scale *
e4m3(code).  Caches are the seeded bf16 paged caches quantised per (page, KV
head) with scale = amax / 448.

The call dequantises the referenced pages to bf16 -- the float32 product
scale * e4m3(code), rounded to nearest bf16 -- before the bf16 paged prefill,
so every case is checked twice:
  * against the bf16 paged-prefill oracle (``oracle.attn_fwd_paged``) on the
    cache dequantised that way, with the forward's bar (``tests/parity.py``):
    this pins the kernels themselves;
  * against the FP8 paged-prefill oracle (``oracle/kv_fp8.py``), which
    dequantises exactly in float64, with the forward's bar widened per row by
    the effect of that one rounding, computed from the data.  With
    delta = max over the sequence's keys of |scale * q . (k_rounded - k)|,
    LSE moves by at most delta (LSE is monotone and shifts with a constant),
    each weight by a factor within exp(+-2 delta), hence O by at most
    max|v_rounded - v| + (exp(2 delta) - 1) * max|v|.
"""
import math

import pytest
import torch

import numpy as np

import oracle
from oracle.kv_fp8 import attn_fwd_paged_fp8 as oracle_paged_fp8
from oracle.kv_fp8 import e4m3_to_float
from exact_softmax_attention_fwd_b200 import attn_fwd_paged_fp8, attn_get_device_error
from exact_softmax_attention_fwd_b200 import workloads as W

from parity import LSE_MAX_ABS, O_MAX_ABS, O_REL_RMS, check, to_f64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _quantised(lens_q, lens_k, Hq, Hkv, d, ps, seed):
    q, cu_q, c = W.paged_prefill_inputs(lens_q, lens_k, Hq, Hkv, d, ps, seed=seed)
    k8, ks = W.quantize_e4m3_per_page(c.k_cache)
    v8, vs = W.quantize_e4m3_per_page(c.v_cache)
    return q, cu_q, k8, v8, ks, vs, c.block_table, c.seq_lens


def _run(q, cu_q, k8, v8, ks, vs, tbl, lens, max_q, causal, scale):
    o, lse = attn_fwd_paged_fp8(q.to(DEV), k8.to(DEV), v8.to(DEV), ks.to(DEV), vs.to(DEV),
                                tbl.to(DEV), cu_q.to(DEV), lens.to(DEV), max_q, causal, scale)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def _dequant_bf16(codes, scales):
    """bf16 cache [pages, page_size, Hkv, d]: the float32 product scale * e4m3(code),
    rounded to nearest bf16 (the call's storage of the dequantised pages)."""
    x = torch.from_numpy(e4m3_to_float(codes.numpy())).float()
    return (x * scales.float()[:, None, :, None]).to(torch.bfloat16)


def _rows_of_keys(cache, tbl, n):
    """The n key rows [n, Hkv, d] of one sequence gathered from a paged cache."""
    ps = cache.shape[1]
    t = torch.arange(n)
    return cache[tbl[t // ps].long(), t % ps]


def _rounding_bounds(q, k8, v8, ks, vs, tbl, cu_q, lens, scale):
    """Per (head, query) row: delta (the largest score shift the bf16 rounding of
    the dequantised keys causes over the sequence's keys), max|v_rounded - v| and
    max|v| over the sequence's values; [Hq, total_q] each."""
    k_ex = torch.from_numpy(e4m3_to_float(k8.numpy())) * ks.double()[:, None, :, None]
    v_ex = torch.from_numpy(e4m3_to_float(v8.numpy())) * vs.double()[:, None, :, None]
    k_rd, v_rd = _dequant_bf16(k8, ks).double(), _dequant_bf16(v8, vs).double()
    total_q, Hq, d = q.shape
    Hkv = k8.shape[2]
    g = Hq // Hkv
    delta = torch.zeros(Hq, total_q, dtype=torch.float64)
    dv = torch.zeros_like(delta)
    vmax = torch.zeros_like(delta)
    for b in range(len(lens)):
        qa, qe, n = int(cu_q[b]), int(cu_q[b + 1]), int(lens[b])
        if qe == qa or n == 0:
            continue
        dk = _rows_of_keys(k_rd, tbl[b], n) - _rows_of_keys(k_ex, tbl[b], n)  # [n, Hkv, d]
        vr, ve = _rows_of_keys(v_rd, tbl[b], n), _rows_of_keys(v_ex, tbl[b], n)
        qq = q[qa:qe].double()                                                # [lq, Hq, d]
        for h in range(Hq):
            kh = h // g
            delta[h, qa:qe] = (scale * qq[:, h] @ dk[:, kh].T).abs().amax(dim=1)
            dv[h, qa:qe] = (vr[:, kh] - ve[:, kh]).abs().max()
            vmax[h, qa:qe] = ve[:, kh].abs().max()
    return delta, dv, vmax


def _check_exact(o, lse, o_ref, lse_ref, bounds, m, what):
    """The forward's bar widened per row by the rounding bounds (module docstring)."""
    delta, dv, vmax = (t[:, m].numpy() for t in bounds)
    og, orf = to_f64(o[m]), np.asarray(o_ref)[m.numpy()]          # [rows, Hq, d]
    lg, lr = to_f64(lse[:, m]), np.asarray(lse_ref)[:, m.numpy()]  # [Hq, rows]
    empty = np.isneginf(lr)
    assert (np.isneginf(lg) == empty).all(), f"{what}: rows disagree on being empty"
    lse_err = np.where(empty, 0.0, np.abs(lg - np.where(empty, 0.0, lr)))
    lse_bar = LSE_MAX_ABS + delta
    assert (lse_err <= lse_bar).all(), f"{what}: LSE off by {(lse_err - lse_bar).max():.3e} over its bar"
    o_extra = (dv + np.expm1(2 * delta) * vmax).T[:, :, None]  # [rows, Hq, 1]
    o_err = np.abs(og - orf)
    assert (o_err <= O_MAX_ABS + o_extra).all(), \
        f"{what}: O off by {(o_err - O_MAX_ABS - o_extra).max():.3e} over its bar"
    rel = np.linalg.norm(og - orf) / np.linalg.norm(orf)
    extra_rel = np.linalg.norm(np.broadcast_to(o_extra, og.shape)) / np.linalg.norm(orf)
    assert rel <= O_REL_RMS + extra_rel, f"{what}: O rel RMS {rel:.3e} > {O_REL_RMS + extra_rel:.3e}"
    return {"lse_max_abs": float(lse_err.max()), "delta_max": float(delta.max()), "o_rel_rms": rel}


def _check_both(o, lse, x, causal, scale, what):
    q, cu_q, k8, v8, ks, vs, tbl, lens = x
    m = _owned(cu_q, q.shape[0])
    # 1. the kernels: bf16 paged prefill of the cache as the call stores it
    o_bf, lse_bf = oracle.attn_fwd_paged(q, _dequant_bf16(k8, ks), _dequant_bf16(v8, vs), tbl,
                                         cu_q, lens, causal, scale)
    check(o[m], o_bf[m.numpy()], lse[:, m], lse_bf[:, m.numpy()], what=f"{what} (bf16 pages)")
    # 2. the format: the exact E4M3 dequantisation, bar widened by the rounding's effect
    o_ref, lse_ref = oracle_paged_fp8(q, k8, v8, ks, vs, tbl, cu_q, lens, causal, scale)
    bounds = _rounding_bounds(q, k8, v8, ks, vs, tbl, cu_q, lens, scale)
    return _check_exact(o, lse, o_ref, lse_ref, bounds, m, what)


def _owned(cu_q, total):
    m = torch.zeros(total, dtype=torch.bool)
    for b in range(len(cu_q) - 1):
        m[int(cu_q[b]):int(cu_q[b + 1])] = True
    return m


MIXES = [
    # (lens_q, lens_k, Hq, Hkv, d, page_size, causal)
    ([100, 1, 300, 129], [700, 1, 300, 1000], 4, 2, 128, 16, True),
    ([256, 0, 77], [2048, 50, 77], 8, 2, 64, 32, True),     # an empty query range
    ([200, 40], [1000, 0], 4, 4, 128, 64, True),            # no cached key at all
    ([130, 600], [4000, 650], 8, 1, 128, 128, False),
]


@pytest.mark.parametrize("case", MIXES, ids=[f"mix{i}" for i in range(len(MIXES))])
def test_paged_prefill_fp8_mixes(case):
    lens_q, lens_k, Hq, Hkv, d, ps, causal = case
    x = _quantised(lens_q, lens_k, Hq, Hkv, d, ps, seed=511)
    scale = 1 / math.sqrt(d)
    o, lse = _run(*x, max(max(lens_q), 1), causal, scale)
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"
    _check_both(o, lse, x, causal, scale, what=f"fp8 paged {case}")


def test_paged_prefill_fp8_gqa_full():
    """The chunked-prefill workload (8 x 1024 new tokens over caches of 0..7168
    tokens, pages of 16, Hq=32, Hkv=8) over its cache quantised to E4M3, every
    token and head."""
    cfg = W.CONFIGS["paged_prefill_gqa"]
    q, cu_q, c, lq, lk = W.paged_prefill_config_inputs(cfg)
    k8, ks = W.quantize_e4m3_per_page(c.k_cache)
    v8, vs = W.quantize_e4m3_per_page(c.v_cache)
    o, lse = _run(q, cu_q, k8, v8, ks, vs, c.block_table, c.seq_lens, int(lq.max()), True,
                  cfg.scale)
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"
    x = (q, cu_q, k8, v8, ks, vs, c.block_table, c.seq_lens)
    _check_both(o, lse, x, True, cfg.scale, what="fp8 paged_prefill_gqa")


def test_paged_prefill_fp8_bad_page_flagged():
    x = list(_quantised([64, 64], [500, 500], 4, 2, 64, 16, seed=513))
    tbl = x[6].clone()
    tbl[0, 3] = x[2].shape[0] + 5  # sequence 0, keys 48..63: a page outside the pool
    x[6] = tbl
    attn_get_device_error()
    o, lse = _run(*x, 64, True, 0.125)
    st, flags = attn_get_device_error()
    assert flags & 0x2, "a page id outside the pool must set ATTN_DEVERR_BAD_PAGE"
    assert torch.isfinite(o.float()).all()
