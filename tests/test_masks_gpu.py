"""GPU parity of attn_fwd_window (sliding-window and prefix-LM masks) against the oracle.

"Attention Kernel", section "可编程 mask": tiles that a row block cannot see
are skipped whole (at both ends for a sliding window) and the tiles left take
an element-wise rule.  Inputs are seeded bf16 on the host; the CUDA path runs
on cuda:0 through the C ABI and the float64 oracle on the same bytes.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_softmax_attention_fwd_b200 import (attn_fwd_masked, attn_fwd_window,
                                             attn_get_device_error, workloads as W)

from parity import check

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _run(q, k, v, scale, window=0, prefix=0, k_lens=None):
    kl = None if k_lens is None else k_lens.to(DEV)
    o, lse = attn_fwd_window(q.to(DEV), k.to(DEV), v.to(DEV), scale, window, prefix, k_lens=kl)
    torch.cuda.synchronize()
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"
    return o.cpu(), lse.cpu()


CASES = [
    # (B, Hq, Hkv, Sq, Sk, d, window, prefix)
    (1, 4, 2, 700, 700, 128, 1, 0),
    (1, 4, 2, 700, 700, 128, 100, 0),
    (2, 2, 1, 513, 513, 64, 128, 0),
    (1, 4, 4, 1000, 1000, 128, 129, 0),
    (1, 2, 2, 300, 900, 128, 256, 0),    # Sq < Sk: windows at the bottom-right diagonal
    (1, 8, 2, 1300, 1300, 128, 1000, 0),
    (1, 4, 2, 700, 700, 128, 0, 1),
    (1, 4, 2, 700, 700, 64, 0, 127),
    (2, 2, 2, 600, 600, 128, 0, 128),
    (1, 4, 1, 900, 900, 128, 0, 333),
    (1, 2, 2, 400, 400, 128, 0, 400),    # prefix covers everything: non-causal
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_window_and_prefix_parity(case):
    B, Hq, Hkv, Sq, Sk, d, window, prefix = case
    q, k, v = W.prefill_inputs(B, Hq, Hkv, Sq, Sk, d, seed=167)
    scale = 1 / math.sqrt(d)
    o, lse = _run(q, k, v, scale, window, prefix)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, True, scale, window=window, prefix=prefix)
    check(o, o_ref, lse, lse_ref, what=f"masks {case}")


def test_window_with_key_padding():
    B, Hq, Hkv, S, d = 3, 4, 2, 600, 128
    q, k, v = W.prefill_inputs(B, Hq, Hkv, S, S, d, seed=173)
    k_lens = torch.tensor([600, 333, 1], dtype=torch.int32)
    o, lse = _run(q, k, v, 0.09, window=200, k_lens=k_lens)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, True, 0.09, k_lens=k_lens, window=200)
    check(o, o_ref, lse, lse_ref, what="window + key padding")


def test_no_mask_and_wide_window_are_the_causal_kernel_bitwise():
    q, k, v = W.prefill_inputs(2, 8, 2, 1111, 1111, 128, seed=179)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    oc, lc = attn_fwd_masked(qd, kd, vd, True, 0.088)
    for window, prefix in ((0, 0), (1111, 0), (5000, 0), (0, 1)):
        ow, lw = attn_fwd_window(qd, kd, vd, 0.088, window, prefix)
        assert torch.equal(oc, ow) and torch.equal(lc, lw), (window, prefix)


def test_sliding_window_8k_sampled_rows():
    c = W.CONFIGS["gqa_causal_8k"]
    q, k, v, _ = W.config_inputs(c)
    o, lse = _run(q, k, v, c.scale, window=1024)
    rows = W.sample_rows(c.B, c.Hq, c.S, 1024, seed=181)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, True, c.scale, rows=rows, window=1024)
    check(o.reshape(-1, c.d)[rows], o_ref, lse.reshape(-1)[rows], lse_ref,
          what="gqa_causal_8k window 1024 sampled rows")


# ------------------------------------------------------------------ block-sparse masks

from exact_softmax_attention_fwd_b200 import attn_fwd_block_sparse  # noqa: E402


def _blocks(B, heads, Sq, Sk, density, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.rand(B, heads, -(-Sq // 128), -(-Sk // 128), generator=g) < density).to(torch.uint8)


def _run_bs(q, k, v, bm, causal, scale, k_lens=None):
    kl = None if k_lens is None else k_lens.to(DEV)
    o, lse = attn_fwd_block_sparse(q.to(DEV), k.to(DEV), v.to(DEV), bm.to(DEV), causal, scale,
                                   k_lens=kl)
    torch.cuda.synchronize()
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"
    return o.cpu(), lse.cpu()


BS_CASES = [
    # (B, Hq, Hkv, Sq, Sk, d, causal, heads, density)
    (1, 4, 2, 700, 700, 128, True, 1, 0.5),
    (2, 4, 4, 513, 900, 64, False, 4, 0.3),
    (1, 8, 2, 1000, 1000, 128, True, 8, 0.7),
    (1, 2, 1, 300, 1300, 128, False, 1, 0.2),
]


@pytest.mark.parametrize("case", BS_CASES, ids=[str(c) for c in BS_CASES])
def test_block_sparse_parity(case):
    B, Hq, Hkv, Sq, Sk, d, causal, heads, density = case
    q, k, v = W.prefill_inputs(B, Hq, Hkv, Sq, Sk, d, seed=199)
    bm = _blocks(B, heads, Sq, Sk, density, seed=211)
    scale = 1 / math.sqrt(d)
    o, lse = _run_bs(q, k, v, bm, causal, scale)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, causal, scale, block_mask=bm)
    check(o, o_ref, lse, lse_ref, what=f"block sparse {case}")


@pytest.mark.parametrize("kind", ["window", "blocks"])
def test_gqa_causal_8k_mask_legs_full(kind):
    """Every element of the two mask workloads bench.py times: the 8k GQA inputs
    (B=2, Hq=32, Hkv=8, S=8192) with a causal sliding window, and with a causal
    block mask shared by the heads (seeded, the bench's density)."""
    import bench

    c = W.CONFIGS["gqa_causal_8k"]
    q, k, v, _ = W.config_inputs(c)
    if kind == "window":
        o, lse = _run(q, k, v, c.scale, window=bench.MASK_WINDOW)
        o_ref, lse_ref = oracle.attn_fwd(q, k, v, True, c.scale, window=bench.MASK_WINDOW)
    else:
        bm = W.block_mask(c.B, 1, c.S, c.S, bench.MASK_DENSITY)
        o, lse = _run_bs(q, k, v, bm, True, c.scale)
        o_ref, lse_ref = oracle.attn_fwd(q, k, v, True, c.scale, block_mask=bm)
    check(o, o_ref, lse, lse_ref, what=f"{c.name} {kind}")


SHARED_CASES = [
    # (B, Hq, Hkv, S, causal, key padding)
    (2, 8, 2, 4096, True, True),     # head-pair units, rows ranked by visible blocks
    (3, 3, 3, 2000, True, False),    # 256-row units of one head, ranked
    (2, 4, 4, 1500, False, True),    # non-causal, ranked
    (13, 2, 1, 8192, True, False),   # 832 unit rows: more than a CTA ranks, causal order kept
]


@pytest.mark.parametrize("case", SHARED_CASES, ids=[str(c) for c in SHARED_CASES])
def test_block_sparse_shared_mask_matches_per_head_copy(case):
    # A mask shared by the heads has its unit rows ranked by their visible
    # blocks in every CTA; the same mask repeated per head keeps the causal
    # ranking.  Each unit is computed the same way whichever CTA takes it, so
    # the two launches must agree bit for bit -- every unit exactly once.
    B, Hq, Hkv, S, causal, padded = case
    q, k, v = W.prefill_inputs(B, Hq, Hkv, S, S, 128, seed=229)
    bm = _blocks(B, 1, S, S, 0.25, seed=233)
    k_lens = None
    if padded:
        g = torch.Generator().manual_seed(239)
        k_lens = torch.randint(S // 2, S + 1, (B,), generator=g, dtype=torch.int32)
    scale = 1 / math.sqrt(128)
    o1, lse1 = _run_bs(q, k, v, bm, causal, scale, k_lens)
    o2, lse2 = _run_bs(q, k, v, bm.expand(B, Hq, -1, -1).contiguous(), causal, scale, k_lens)
    assert torch.equal(o1, o2) and torch.equal(lse1, lse2)
    assert bool(torch.isfinite(o1).all())


def test_block_sparse_band_with_key_padding():
    B, Hq, Hkv, S, d = 2, 4, 2, 900, 128
    q, k, v = W.prefill_inputs(B, Hq, Hkv, S, S, d, seed=223)
    n = -(-S // 128)
    t = torch.arange(n)
    bm = ((t[:, None] - t[None, :]).abs() <= 1).to(torch.uint8).view(1, 1, n, n).repeat(B, 1, 1, 1)
    k_lens = torch.tensor([900, 400], dtype=torch.int32)
    o, lse = _run_bs(q, k, v, bm, True, 0.09, k_lens)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, True, 0.09, k_lens=k_lens, block_mask=bm)
    check(o, o_ref, lse, lse_ref, what="block band + key padding")


def test_block_sparse_all_ones_bitwise_and_empty_tiles():
    q, k, v = W.prefill_inputs(1, 4, 2, 600, 600, 128, seed=227)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    for causal in (False, True):
        ones = torch.ones(1, 1, 5, 5, dtype=torch.uint8, device=DEV)
        a = attn_fwd_masked(qd, kd, vd, causal, 0.1)
        b = attn_fwd_block_sparse(qd, kd, vd, ones, causal, 0.1)
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]), causal
    bm = torch.ones(1, 4, 5, 5, dtype=torch.uint8)
    bm[0, 2, 1, :] = 0  # head 2, query rows 128..255: nothing visible
    bm[0, 1, :, 0] = 0
    o, lse = _run_bs(q, k, v, bm, False, 0.1)
    assert torch.all(o[0, 2, 128:256] == 0) and torch.isneginf(lse[0, 2, 128:256]).all()
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, False, 0.1, block_mask=bm)
    check(o, o_ref, lse, lse_ref, what="block sparse with empty tiles")
