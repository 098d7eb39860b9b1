"""Seeded random sweeps of small shapes through the E4M3 paths: the
block-scaled prefill and the paged decode over an E4M3 cache, each case
against the float64 FP8 oracles on the same codes and scales, with the
forward's bar (``tests/parity.py``) as their own tests hold them.  Values are
drawn as the named workloads draw them (N(0,1) x 0.5) before quantisation.
"""
import math
import random

import pytest
import torch

from oracle.kv_fp8 import attn_fwd_fp8 as oracle_fwd_fp8
from oracle.kv_fp8 import decode_paged_fp8 as oracle_decode_fp8
from exact_softmax_attention_fwd_b200 import (attn_decode_paged_fp8, attn_fwd_fp8,
                                             attn_get_device_error)
from exact_softmax_attention_fwd_b200 import workloads as W

from parity import check

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
N_CASES = 16


def _device_ok():
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"


def _len(rng, lo, hi):
    if rng.random() < 0.5:
        base = rng.choice([128, 256, 384, 512])
        return max(lo, min(hi, base + rng.choice([-1, 0, 1])))
    return rng.randint(lo, hi)


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_fp8_prefill(case):
    rng = random.Random(9000 + case)
    hkv = rng.choice([1, 2, 4])
    Hq, Hkv = hkv * rng.choice([1, 2, 4]), hkv
    B = rng.randint(1, 2)
    Sq, Sk = _len(rng, 1, 700), _len(rng, 1, 700)
    causal = rng.random() < 0.6
    scale = 1.0 / math.sqrt(128)
    x = W.fp8_prefill_inputs(B, Hq, Hkv, Sq, Sk, 128, seed=9100 + case, value_scale=0.5)
    k_lens = None
    if rng.random() < 0.4:
        k_lens = torch.tensor([rng.randint(0, Sk) for _ in range(B)], dtype=torch.int32)
    kl = None if k_lens is None else k_lens.to(DEV)
    o, lse = attn_fwd_fp8(*(t.to(DEV) for t in x), causal, scale, k_lens=kl)
    torch.cuda.synchronize()
    _device_ok()
    o_ref, lse_ref = oracle_fwd_fp8(*x, causal, scale,
                                    k_lens=None if k_lens is None else k_lens.numpy())
    check(o.cpu(), o_ref, lse.cpu(), lse_ref,
          what=f"fp8 prefill B{B} Hq{Hq} Hkv{Hkv} Sq{Sq} Sk{Sk} c{causal} kl{k_lens}")


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_fp8_decode(case):
    rng = random.Random(9200 + case)
    hkv = rng.choice([1, 2, 4, 8])
    Hq, Hkv = hkv * rng.choice([1, 2, 4, 8]), hkv
    B = rng.randint(1, 8)
    ps = rng.choice([16, 32, 64])
    lens = [rng.choice([0, rng.randint(1, 40), rng.randint(500, 530), rng.randint(1, 2100)])
            for _ in range(B)]
    d = rng.choice([64, 128])
    scale = 1.0 / math.sqrt(d)
    c = W.fp8_paged_inputs(torch.tensor(lens, dtype=torch.int32), Hq, Hkv, d, ps,
                           seed=9300 + case, extra_pages=rng.randint(0, 2))
    o, lse = attn_decode_paged_fp8(c.q.to(DEV), c.k_cache.to(DEV), c.v_cache.to(DEV),
                                   c.k_scale.to(DEV), c.v_scale.to(DEV), c.block_table.to(DEV),
                                   c.seq_lens.to(DEV), scale)
    torch.cuda.synchronize()
    _device_ok()
    o_ref, lse_ref = oracle_decode_fp8(c.q, c.k_cache, c.v_cache, c.k_scale, c.v_scale,
                                       c.block_table, c.seq_lens, scale)
    check(o.cpu(), o_ref, lse.cpu(), lse_ref,
          what=f"fp8 decode lens{lens} Hq{Hq} Hkv{Hkv} d{d} p{ps}")
