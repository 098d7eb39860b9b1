"""GPU parity of attn_bwd_window and attn_bwd_block_sparse (the backward of the
programmable-mask forwards) against the float64 backward oracle.

"Attention Kernel", section "Backward 与重计算": the backward applies the
forward's mask unchanged; section "可编程 mask": sliding window, prefix-LM and
block-level sparsity.  O and LSE come from the CUDA masked forwards; the
oracle (``oracle/attn_bwd.py``) forms the masked probabilities from the
definition.  Gradients are compared element by element (``tests/parity.py``).
"""
import math

import numpy as np
import pytest
import torch

from oracle.attn_bwd import attn_bwd as oracle_bwd
from exact_softmax_attention_fwd_b200 import (attn_bwd_block_sparse, attn_bwd_window,
                                             attn_fwd_block_sparse, attn_fwd_window,
                                             attn_get_device_error, workloads as W)

from parity import check_grad

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _check(got, ref, what):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        if not np.any(r):
            # A gradient that vanishes by cancellation, not for want of a visible
            # pair (a window of 1: each row's weight is 1, so dS = dP - D = 0 in
            # exact arithmetic): the kernel forms D from the bf16-rounded O, so
            # it is zero only to rounding.
            assert float(g.float().abs().max()) <= 1e-3, f"{what} {name}"
            continue
        check_grad(g.cpu(), r, what=f"{what} {name}")


WINDOWS = [
    # B, Hq, Hkv, Sq, Sk, d, window, prefix
    (1, 4, 2, 700, 700, 128, 200, 0),
    (1, 2, 2, 512, 512, 64, 1, 0),        # window 1: each row's diagonal key only
    (2, 4, 1, 300, 700, 128, 256, 0),     # Sq < Sk: bottom-right window
    (1, 4, 2, 600, 600, 128, 0, 130),     # prefix-LM
    (1, 2, 1, 400, 250, 64, 0, 100),      # Sq > Sk: leading rows see only the prefix
]


@pytest.mark.parametrize("case", WINDOWS, ids=[str(c) for c in WINDOWS])
def test_bwd_window_and_prefix(case):
    B, Hq, Hkv, Sq, Sk, d, window, prefix = case
    q, k, v = W.prefill_inputs(B, Hq, Hkv, Sq, Sk, d, seed=401 + Sq + window + prefix)
    do = W.grad_output(B, Hq, Sq, d, seed=401 + Sq)
    scale = 1 / math.sqrt(d)
    qd, kd, vd, dod = (x.to(DEV) for x in (q, k, v, do))
    o, lse = attn_fwd_window(qd, kd, vd, scale, window=window, prefix=prefix)
    got = attn_bwd_window(qd, kd, vd, o, lse, dod, scale, window=window, prefix=prefix)
    torch.cuda.synchronize()
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"
    ref = oracle_bwd(q, k, v, do, True, scale, window=window, prefix=prefix)
    _check(got, ref, f"window {case}")


def test_bwd_window_with_key_padding():
    B, Hq, Hkv, S, d = 3, 4, 2, 500, 128
    q, k, v = W.prefill_inputs(B, Hq, Hkv, S, S, d, seed=411)
    do = W.grad_output(B, Hq, S, d, seed=411)
    k_lens = torch.tensor([500, 333, 0], dtype=torch.int32)
    qd, kd, vd, dod = (x.to(DEV) for x in (q, k, v, do))
    o, lse = attn_fwd_window(qd, kd, vd, 0.088, window=150, k_lens=k_lens.to(DEV))
    got = attn_bwd_window(qd, kd, vd, o, lse, dod, 0.088, window=150, k_lens=k_lens.to(DEV))
    torch.cuda.synchronize()
    ref = oracle_bwd(q, k, v, do, True, 0.088, k_lens=k_lens.numpy(), window=150)
    _check(got, ref, "window + padding")


BLOCKS = [
    # B, Hq, Hkv, Sq, Sk, d, causal, per_head
    (1, 4, 2, 640, 640, 128, True, True),
    (2, 2, 2, 384, 512, 128, False, False),
    (1, 4, 1, 300, 700, 64, True, True),
]


@pytest.mark.parametrize("case", BLOCKS, ids=[str(c) for c in BLOCKS])
def test_bwd_block_sparse(case):
    B, Hq, Hkv, Sq, Sk, d, causal, per_head = case
    q, k, v = W.prefill_inputs(B, Hq, Hkv, Sq, Sk, d, seed=421 + Sq)
    do = W.grad_output(B, Hq, Sq, d, seed=421 + Sq)
    nq, nk = -(-Sq // 128), -(-Sk // 128)
    g = torch.Generator().manual_seed(423 + Sq)
    mask = (torch.rand(B, Hq if per_head else 1, nq, nk, generator=g) < 0.5).to(torch.uint8)
    mask[:, :, 0, :] = 0  # a query tile with no block at all: zero dQ, no gradient from it
    mask[:, :, :, 1] = 0  # a key tile no query tile keeps: its dK / dV units walk nothing
    scale = 1 / math.sqrt(d)
    qd, kd, vd, dod, md = (x.to(DEV) for x in (q, k, v, do, mask))
    o, lse = attn_fwd_block_sparse(qd, kd, vd, md, causal, scale)
    got = attn_bwd_block_sparse(qd, kd, vd, o, lse, dod, md, causal, scale)
    torch.cuda.synchronize()
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"
    ref = oracle_bwd(q, k, v, do, causal, scale, block_mask=mask.numpy())
    _check(got, ref, f"blocks {case}")
    assert not got[0][:, :, :128].float().abs().sum()  # rows of the empty query tile
    assert not got[1][:, :, 128:256].float().abs().sum()  # rows of the empty key tile
    assert not got[2][:, :, 128:256].float().abs().sum()


def test_bwd_all_ones_block_mask_equals_plain_backward():
    from exact_softmax_attention_fwd_b200 import attn_bwd, attn_fwd_masked
    B, Hq, Hkv, S, d = 1, 4, 2, 384, 128
    q, k, v = (x.to(DEV) for x in W.prefill_inputs(B, Hq, Hkv, S, S, d, seed=431))
    do = W.grad_output(B, Hq, S, d, seed=431).to(DEV)
    o, lse = attn_fwd_masked(q, k, v, True, 0.088)
    ones = torch.ones(B, 1, 3, 3, dtype=torch.uint8, device=DEV)
    a = attn_bwd(q, k, v, o, lse, do, True, 0.088)
    b = attn_bwd_block_sparse(q, k, v, o, lse, do, ones, True, 0.088)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
