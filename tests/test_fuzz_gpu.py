"""Seeded random sweeps of small shapes through every forward entry point,
each case against the float64 oracle on the same bytes.

The named workloads and the hand-picked edge cases elsewhere check the paths
at their sizes; these sweeps draw head counts, group sizes, lengths that
straddle tile and split boundaries, key padding, causal or not, head
dimension, page sizes and scales from a fixed seed, so that the index
arithmetic of every kernel meets shapes nobody chose by hand.  The bar is the
forward's (``tests/parity.py``), and the dense and ragged sweeps draw their
values as the named workloads do (N(0,1) x 0.5): the bar's 1e-2 on the largest error of O
assumes outputs below about 2, where half a bf16 step is 4e-3; with softmax
scale 0.5 and N(0,1) values the output is nearly a single value row of up to
about 4, and the rounding of O to bf16 alone reaches 8e-3.
"""
import math
import random

import pytest
import torch

import oracle
from exact_softmax_attention_fwd_b200 import (attn_decode_paged, attn_fwd_masked, attn_fwd_paged,
                                             attn_fwd_varlen, attn_get_device_error)
from exact_softmax_attention_fwd_b200 import workloads as W

from parity import check

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
N_CASES = 24


def _heads(rng):
    hkv = rng.choice([1, 2, 3, 4])
    return hkv * rng.choice([1, 2, 4, 8]), hkv


def _len(rng, lo, hi):
    # lengths near tile (128) and unit (256) boundaries are drawn more often
    if rng.random() < 0.5:
        base = rng.choice([128, 256, 384, 512])
        return max(lo, min(hi, base + rng.choice([-1, 0, 1])))
    return rng.randint(lo, hi)


def _device_ok():
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"


def _owned(cu_q, total):
    m = torch.zeros(total, dtype=torch.bool)
    for b in range(len(cu_q) - 1):
        m[int(cu_q[b]):int(cu_q[b + 1])] = True
    return m


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_dense_prefill(case):
    rng = random.Random(7000 + case)
    Hq, Hkv = _heads(rng)
    B = rng.randint(1, 3)
    Sq, Sk = _len(rng, 1, 700), _len(rng, 0, 700)
    d = rng.choice([64, 128])
    causal = rng.random() < 0.6
    scale = rng.choice([1.0 / math.sqrt(d), 0.5, 0.05])
    q, k, v = W.prefill_inputs(B, Hq, Hkv, Sq, Sk, d, seed=7100 + case, value_scale=0.5)
    k_lens = None
    if Sk > 0 and rng.random() < 0.5:
        k_lens = torch.tensor([rng.randint(0, Sk) for _ in range(B)], dtype=torch.int32)
    kl = None if k_lens is None else k_lens.to(DEV)
    o, lse = attn_fwd_masked(q.to(DEV), k.to(DEV), v.to(DEV), causal, scale, k_lens=kl)
    torch.cuda.synchronize()
    _device_ok()
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, causal, scale, k_lens=k_lens)
    check(o.cpu(), o_ref, lse.cpu(), lse_ref,
          what=f"dense B{B} Hq{Hq} Hkv{Hkv} Sq{Sq} Sk{Sk} d{d} c{causal} kl{k_lens}")


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_ragged_prefill(case):
    rng = random.Random(7200 + case)
    Hq, Hkv = _heads(rng)
    B = rng.randint(1, 5)
    lens_q = [_len(rng, 0, 600) for _ in range(B)]
    same = rng.random() < 0.5
    lens_k = list(lens_q) if same else [_len(rng, 0, 600) for _ in range(B)]
    d = rng.choice([64, 128])
    causal = rng.random() < 0.6
    scale = 1.0 / math.sqrt(d)
    q, k, v, cu_q, cu_k = W.varlen_inputs(lens_q, lens_k, Hq, Hkv, d, seed=7300 + case,
                                         value_scale=0.5)
    max_q = max(max(lens_q), 1)
    o, lse = attn_fwd_varlen(q.to(DEV), k.to(DEV), v.to(DEV), cu_q.to(DEV), cu_k.to(DEV), max_q,
                             causal, scale)
    torch.cuda.synchronize()
    _device_ok()
    o_ref, lse_ref = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, causal, scale)
    m = _owned(cu_q, q.shape[0])
    check(o.cpu()[m], o_ref[m.numpy()], lse.cpu()[:, m], lse_ref[:, m.numpy()],
          what=f"ragged q{lens_q} k{lens_k} Hq{Hq} Hkv{Hkv} d{d} c{causal}")


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_paged_prefill(case):
    rng = random.Random(7400 + case)
    Hq, Hkv = _heads(rng)
    B = rng.randint(1, 4)
    ps = rng.choice([16, 32, 64, 128])
    lens_q = [_len(rng, 0, 400) for _ in range(B)]
    lens_k = [lq + _len(rng, 0, 500) for lq in lens_q]  # an append: keys include the queries
    d = rng.choice([64, 128])
    causal = rng.random() < 0.7
    scale = 1.0 / math.sqrt(d)
    q, cu_q, c = W.paged_prefill_inputs(lens_q, lens_k, Hq, Hkv, d, ps, seed=7500 + case)
    max_q = max(max(lens_q), 1)
    o, lse = attn_fwd_paged(q.to(DEV), c.k_cache.to(DEV), c.v_cache.to(DEV),
                            c.block_table.to(DEV), cu_q.to(DEV), c.seq_lens.to(DEV), max_q,
                            causal, scale)
    torch.cuda.synchronize()
    _device_ok()
    o_ref, lse_ref = oracle.attn_fwd_paged(q, c.k_cache, c.v_cache, c.block_table, cu_q,
                                           c.seq_lens, causal, scale)
    m = _owned(cu_q, q.shape[0])
    check(o.cpu()[m], o_ref[m.numpy()], lse.cpu()[:, m], lse_ref[:, m.numpy()],
          what=f"paged q{lens_q} k{lens_k} Hq{Hq} Hkv{Hkv} d{d} p{ps} c{causal}")


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_decode(case):
    rng = random.Random(7600 + case)
    hkv = rng.choice([1, 2, 4, 8])
    Hq, Hkv = hkv * rng.choice([1, 2, 4, 8]), hkv
    B = rng.randint(1, 9)
    ps = rng.choice([16, 32, 64])
    # lengths around the 512-token split and the page boundaries, and empty ones
    lens = [rng.choice([0, rng.randint(1, 40), rng.randint(500, 530), rng.randint(1, 2100)])
            for _ in range(B)]
    d = rng.choice([64, 128])
    scale = 1.0 / math.sqrt(d)
    inp = W.paged_inputs(torch.tensor(lens, dtype=torch.int32), Hq, Hkv, d, ps, seed=7700 + case,
                         extra_pages=rng.randint(0, 3))
    o, lse = attn_decode_paged(inp.q.to(DEV), inp.k_cache.to(DEV), inp.v_cache.to(DEV),
                               inp.block_table.to(DEV), inp.seq_lens.to(DEV), scale)
    torch.cuda.synchronize()
    _device_ok()
    o_ref, lse_ref = oracle.decode_paged(inp.q, inp.k_cache, inp.v_cache, inp.block_table,
                                         inp.seq_lens, scale)
    check(o.cpu(), o_ref, lse.cpu(), lse_ref,
          what=f"decode lens{lens} Hq{Hq} Hkv{Hkv} d{d} p{ps}")
