"""GPU parity of attn_fwd_paged_fp8 (packed queries appended to an E4M3 paged
cache) against the FP8 paged-prefill oracle.

"Attention Kernel", sections "Paged 与 ragged KV" and "正确性契约": the cache
holds E4M3 codes with one scale per (page, KV head), element = scale *
e4m3(code).  Caches are the seeded bf16 paged caches quantised per (page, KV
head) with scale = amax / 448; the oracle (``oracle/kv_fp8.py``,
``attn_fwd_paged_fp8``) dequantises them from the format's definition.  The
call dequantises the referenced pages to bf16 (one rounding of scale * value)
before the bf16 paged prefill; a float64 model of that rounding alone gives
rel-RMS 2.4e-3 on a 2,000-key mix, inside the forward's bar with the kernel's
own rounding of P, so the forward's bar (``tests/parity.py``) applies.
"""
import math

import pytest
import torch

from oracle.kv_fp8 import attn_fwd_paged_fp8 as oracle_paged_fp8
from exact_softmax_attention_fwd_b200 import attn_fwd_paged_fp8, attn_get_device_error
from exact_softmax_attention_fwd_b200 import workloads as W

from parity import check

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
    q, cu_q, k8, v8, ks, vs, tbl, lens = x
    o_ref, lse_ref = oracle_paged_fp8(q, k8, v8, ks, vs, tbl, cu_q, lens, causal, scale)
    m = _owned(cu_q, q.shape[0])
    check(o[m], o_ref[m.numpy()], lse[:, m], lse_ref[:, m.numpy()], what=f"fp8 paged {case}")


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
    o_ref, lse_ref = oracle_paged_fp8(q, k8, v8, ks, vs, c.block_table, cu_q, c.seq_lens, True,
                                      cfg.scale)
    check(o, o_ref, lse, lse_ref, what="fp8 paged_prefill_gqa")


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
