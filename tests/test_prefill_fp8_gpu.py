"""GPU parity of attn_fwd_fp8 (prefill over block-scaled E4M3 Q, K, V) against
the FP8 prefill oracle.

"Attention 算子加速史", section 3.3: FP8 operands with block-level scaling.
Inputs are the seeded bf16 workloads quantised per (batch, head, 128-row block)
with scale = amax / 448 (``workloads.quantize_e4m3_blocks``); the CUDA path
gets the codes and scales, the float64 oracle (``oracle/kv_fp8.py``,
``attn_fwd_fp8``) the same bytes, dequantised from the format's definition.
The comparison uses the forward's bar (``tests/parity.py``): the kernel's
score products of E4M3 codes are exact, V is widened exactly (to f16), and
the weights, scaled by each V block's scale over the largest one, are rounded
to f16 for the P.V product.
"""
import math

import pytest
import torch

from oracle.kv_fp8 import attn_fwd_fp8 as oracle_fp8
from exact_softmax_attention_fwd_b200 import attn_fwd_fp8, attn_get_device_error
from exact_softmax_attention_fwd_b200 import workloads as W

from parity import check

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _run(q8, k8, v8, qs, ks, vs, causal, scale, k_lens=None):
    dv = [t.to(DEV) for t in (q8, k8, v8, qs, ks, vs)]
    kl = None if k_lens is None else k_lens.to(DEV)
    o, lse = attn_fwd_fp8(*dv, causal, scale, k_lens=kl)
    torch.cuda.synchronize()
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"
    return o.cpu(), lse.cpu()


CASES = [
    # B, Hq, Hkv, Sq, Sk, causal
    (1, 2, 2, 256, 256, False),
    (1, 4, 2, 300, 300, True),     # ragged tail
    (2, 4, 1, 129, 517, True),     # Sq < Sk: bottom-right diagonal
    (2, 2, 2, 300, 100, True),     # Sq > Sk: leading rows see no key
    (1, 8, 2, 640, 640, False),    # GQA, several key tiles
    (1, 2, 2, 1024, 1024, True),
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_fp8_prefill_cases(case):
    B, Hq, Hkv, Sq, Sk, causal = case
    x = W.fp8_prefill_inputs(B, Hq, Hkv, Sq, Sk, 128, seed=301 + Sq + Sk)
    scale = 1 / math.sqrt(128)
    o, lse = _run(*x, causal, scale)
    o_ref, lse_ref = oracle_fp8(*x, causal, scale)
    check(o, o_ref, lse, lse_ref, what=f"fp8 prefill {case}")


def test_fp8_prefill_mha_causal_2k_full():
    """The 2k causal workload's shapes (B=4, H=16, S=2048), quantised, every element."""
    c = W.CONFIGS["mha_causal_2k"]
    x = W.fp8_prefill_inputs(c.B, c.Hq, c.Hkv, c.S, c.S, c.d, seed=c.seed)
    o, lse = _run(*x, True, c.scale)
    o_ref, lse_ref = oracle_fp8(*x, True, c.scale)
    check(o, o_ref, lse, lse_ref, what="fp8 mha_causal_2k")


def test_fp8_prefill_gqa_causal_8k_two_kv_groups():
    """The launch the bench times: the gqa_causal_8k inputs (B=2, Hq=32, Hkv=8,
    S=8192, causal) quantised and run whole.  Checked: the first and the last
    1024 query rows of two KV-head groups (batch 0 / KV head 0 and batch 1 /
    KV head 7, four query heads each), every element, against the oracle run
    on those rows alone -- the first rows see only the first 1024 keys, the
    last rows all 8192 keys with the bottom-right causal rule, and both
    slices start on a 128-row block, so their scales are the launch's own."""
    c = W.CONFIGS["gqa_causal_8k"]
    x = W.fp8_prefill_inputs(c.B, c.Hq, c.Hkv, c.S, c.S, c.d, c.seed, c.value_scale)
    o, lse = _run(*x, True, c.scale)
    q8, k8, v8, qs, ks, vs = x
    g, S, R = c.Hq // c.Hkv, c.S, 1024
    for b, kvh in ((0, 0), (c.B - 1, c.Hkv - 1)):
        bb, hs, kv = slice(b, b + 1), slice(kvh * g, (kvh + 1) * g), slice(kvh, kvh + 1)
        last, last_blk = slice(S - R, S), slice((S - R) // 128, S // 128)
        o_ref, lse_ref = oracle_fp8(q8[bb, hs, last], k8[bb, kv], v8[bb, kv], qs[bb, hs, last_blk],
                                    ks[bb, kv], vs[bb, kv], True, c.scale)
        check(o[bb, hs, last], o_ref, lse[bb, hs, last], lse_ref,
              what=f"fp8 gqa_causal_8k batch {b} KV head {kvh}, last {R} rows")
        first, first_blk = slice(0, R), slice(0, R // 128)
        o_ref, lse_ref = oracle_fp8(q8[bb, hs, first], k8[bb, kv, first], v8[bb, kv, first],
                                    qs[bb, hs, first_blk], ks[bb, kv, first_blk],
                                    vs[bb, kv, first_blk], True, c.scale)
        check(o[bb, hs, first], o_ref, lse[bb, hs, first], lse_ref,
              what=f"fp8 gqa_causal_8k batch {b} KV head {kvh}, first {R} rows")


def test_fp8_prefill_key_padding_and_empty_rows():
    x = W.fp8_prefill_inputs(3, 4, 2, 256, 256, 128, seed=303)
    k_lens = torch.tensor([0, 77, 256], dtype=torch.int32)
    o, lse = _run(*x, True, 0.088, k_lens=k_lens)
    o_ref, lse_ref = oracle_fp8(*x, True, 0.088, k_lens=k_lens)
    stats = check(o, o_ref, lse, lse_ref, what="fp8 padding")
    assert stats["empty_rows"] > 0
    assert torch.all(o[0] == 0) and torch.all(torch.isneginf(lse[0]))


@pytest.mark.parametrize("scale", [0.0, -0.2])
def test_fp8_prefill_unusual_scales(scale):
    x = W.fp8_prefill_inputs(1, 2, 1, 300, 300, 128, seed=305)
    o, lse = _run(*x, True, scale)
    o_ref, lse_ref = oracle_fp8(*x, True, scale)
    check(o, o_ref, lse, lse_ref, what=f"fp8 scale {scale}")


def test_fp8_prefill_deterministic():
    x = W.fp8_prefill_inputs(2, 4, 2, 700, 700, 128, seed=307)
    a = _run(*x, True, 0.088)
    b = _run(*x, True, 0.088)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_fp8_prefill_v_block_scales_far_apart():
    """V block scales twelve orders of magnitude apart, and one of zero: such a
    block's weights underflow f16 in the P.V product, but they still count in
    the normaliser (its values are ~0, its attention mass is not)."""
    B, Hq, Hkv, S = 1, 4, 2, 600
    q8, k8, v8, qs, ks, vs = W.fp8_prefill_inputs(B, Hq, Hkv, S, S, 128, seed=311)
    vs = vs.clone()
    vs[:, :, 1] = 1e-12
    vs[:, 0, 3] = 0.0
    for causal in (True, False):
        o, lse = _run(q8, k8, v8, qs, ks, vs, causal, 0.088)
        o_ref, lse_ref = oracle_fp8(q8, k8, v8, qs, ks, vs, causal, 0.088)
        check(o, o_ref, lse, lse_ref, what=f"fp8 V scales far apart causal={causal}")
