"""GPU parity of attn_decode_paged_fp8 (decode over an E4M3 paged cache with a
scale per (page, KV head)) against the float64 FP8-cache oracle.

"Attention Kernel", section "正确性契约": the cache quantisation schema is
part of the contract; the oracle dequantises by the E4M3 definition and the
scales, then attends exactly.  Inputs are a seeded bf16 cache quantised per
page (scale = amax / 448), on the host; the CUDA path runs through the C ABI.
"""
import math

import numpy as np
import pytest
import torch

from oracle.kv_fp8 import decode_paged_fp8 as oracle_fp8
from exact_softmax_attention_fwd_b200 import attn_decode_paged_fp8, attn_get_device_error
from exact_softmax_attention_fwd_b200 import workloads as W

from parity import check

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _run(c, scale):
    o, lse = attn_decode_paged_fp8(c.q.to(DEV), c.k_cache.to(DEV), c.v_cache.to(DEV),
                                   c.k_scale.to(DEV), c.v_scale.to(DEV), c.block_table.to(DEV),
                                   c.seq_lens.to(DEV), scale)
    torch.cuda.synchronize()
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"
    return o.cpu(), lse.cpu()


def _ref(c, scale):
    return oracle_fp8(c.q, c.k_cache, c.v_cache, c.k_scale, c.v_scale, c.block_table, c.seq_lens,
                      scale)


CASES = [
    # lens, Hq, Hkv, d, page_size
    ([1, 2, 15, 16, 17, 31, 32, 33], 32, 8, 128, 16),
    ([0, 5, 0, 600], 8, 2, 128, 16),                     # empty sequences
    ([511, 512, 513, 1024, 1025, 1500], 4, 4, 128, 16),  # split boundaries (g = 1)
    ([700, 33, 4096], 16, 2, 128, 16),                   # g = 8
    ([300, 1, 64], 8, 4, 64, 16),                        # d = 64, g = 2
    ([100, 257, 1000], 8, 2, 128, 32),                   # page size 32
    ([129, 800], 6, 3, 64, 64),                          # page size 64, odd heads
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_fp8_decode_cases(case):
    lens, Hq, Hkv, d, ps = case
    c = W.fp8_paged_inputs(torch.tensor(lens, dtype=torch.int32), Hq, Hkv, d, ps, seed=41,
                           extra_pages=2)
    scale = 1 / math.sqrt(d)
    o, lse = _run(c, scale)
    o_ref, lse_ref = _ref(c, scale)
    check(o, o_ref, lse, lse_ref, what=f"fp8 {case}")


def test_fp8_decode_config_full():
    """The paged_decode workload (B=64, Hq=32, Hkv=8, d=128, page 16, lengths
    U[512, 8192]) with its cache quantised to E4M3, every output checked."""
    cfg = W.CONFIGS["paged_decode"]
    base = W.decode_config_inputs(cfg)
    k8, ks = W.quantize_e4m3_per_page(base.k_cache)
    v8, vs = W.quantize_e4m3_per_page(base.v_cache)
    c = W.PagedFp8Inputs(base.q, k8, v8, ks, vs, base.block_table, base.seq_lens, cfg.page_size)
    o, lse = _run(c, cfg.scale)
    o_ref, lse_ref = _ref(c, cfg.scale)
    check(o, o_ref, lse, lse_ref, what="fp8 paged_decode")


def test_fp8_scales_are_per_page_and_head():
    """Scaling one page's V scale by 4 changes only what that page contributes:
    the GPU follows the oracle on the modified scales, and the output moves."""
    c = W.fp8_paged_inputs(torch.tensor([200, 90], dtype=torch.int32), 8, 2, 128, 16, seed=42)
    scale = 1 / math.sqrt(128)
    o0, _ = _run(c, scale)
    page = int(c.block_table[0, 3])
    c.v_scale[page, 1] *= 4.0
    c.k_scale[page, 0] *= 0.5
    o1, lse1 = _run(c, scale)
    o_ref, lse_ref = _ref(c, scale)
    check(o1, o_ref, lse1, lse_ref, what="modified page scales")
    assert not torch.equal(o0[0, 4:8], o1[0, 4:8])  # heads of KV head 1 in sequence 0
    assert torch.equal(o0[1], o1[1])                 # sequence 1 does not use that page


def test_fp8_decode_deterministic_and_bad_page_flagged():
    c = W.fp8_paged_inputs(torch.tensor([1000, 17], dtype=torch.int32), 8, 2, 128, 16, seed=43)
    a, _ = _run(c, 0.1)
    b, _ = _run(c, 0.1)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    c.block_table[0, 5] = c.num_pages + 7  # out of range: skipped and flagged
    attn_decode_paged_fp8(c.q.to(DEV), c.k_cache.to(DEV), c.v_cache.to(DEV), c.k_scale.to(DEV),
                          c.v_scale.to(DEV), c.block_table.to(DEV), c.seq_lens.to(DEV), 0.1)
    st, flags = attn_get_device_error()
    assert st != 0 and flags & 0x2


def test_fp8_slots_past_the_length_never_reach_the_result():
    """As for the bf16 cache: unused slots of the last page may hold the E4M3
    NaN code (0x7F) without changing a bit of the result."""
    c = W.fp8_paged_inputs(torch.tensor([37, 500, 16], dtype=torch.int32), 8, 2, 128, 16,
                           seed=44)
    o1, l1 = _run(c, 0.088)
    kc, vc = c.k_cache.clone(), c.v_cache.clone()
    for b, n in enumerate(c.seq_lens.tolist()):
        last = int(c.block_table[b, (n - 1) // 16])
        kc[last, n % 16 or 16:] = 0x7F
        vc[last, n % 16 or 16:] = 0x7F
    c2 = W.PagedFp8Inputs(c.q, kc, vc, c.k_scale, c.v_scale, c.block_table, c.seq_lens, 16)
    o2, l2 = _run(c2, 0.088)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fp8_scales_of_any_sign_and_zero():
    """The schema allows any finite scale: negative K and V scales flip the
    sign of a page's scores or values, and a zero V scale removes a page's
    values but not its weights from the softmax.  GPU against the oracle on
    the same scales, with pages of each kind inside one split and across
    splits (lengths up to 1300 tokens: three 512-token splits)."""
    c = W.fp8_paged_inputs(torch.tensor([1300, 97, 530], dtype=torch.int32), 8, 2, 128, 16,
                           seed=43)
    scale = 1 / math.sqrt(128)
    g = torch.Generator().manual_seed(44)
    ks, vs = c.k_scale.clone(), c.v_scale.clone()
    flip_k = torch.rand(ks.shape, generator=g) < 0.3
    flip_v = torch.rand(vs.shape, generator=g) < 0.3
    zero_v = torch.rand(vs.shape, generator=g) < 0.15
    ks[flip_k] = -ks[flip_k]
    vs[flip_v] = -vs[flip_v]
    vs[zero_v] = 0.0
    c2 = W.PagedFp8Inputs(c.q, c.k_cache, c.v_cache, ks, vs, c.block_table, c.seq_lens,
                          c.page_size)
    o, lse = _run(c2, scale)
    o_ref, lse_ref = _ref(c2, scale)
    check(o, o_ref, lse, lse_ref, what="fp8 scales of any sign")
