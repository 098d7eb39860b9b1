"""Seeded random sweeps of small shapes through the programmable-mask forwards
and every backward entry point, each case against the float64 oracles.

As in ``test_fuzz_gpu.py``: head counts, group sizes, lengths near tile
boundaries, key padding, windows, prefixes and block densities are drawn from
a fixed seed, values as the named workloads draw them (N(0,1) x 0.5).
Forward outputs meet the forward's bar, gradients the backward's
(``tests/parity.py``); a gradient that vanishes by cancellation is held to
rounding (1e-3), as in the masked-backward tests.
"""
import math
import random

import numpy as np
import pytest
import torch

import oracle
from oracle.attn_bwd import attn_bwd as oracle_bwd
from oracle.attn_bwd import attn_bwd_varlen as oracle_bwd_varlen
from exact_softmax_attention_fwd_b200 import (attn_bwd, attn_bwd_block_sparse, attn_bwd_varlen,
                                             attn_bwd_window, attn_fwd_block_sparse,
                                             attn_fwd_masked, attn_fwd_varlen, attn_fwd_window,
                                             attn_get_device_error)
from exact_softmax_attention_fwd_b200 import workloads as W

from parity import check, check_grad

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
N_CASES = 16


def _heads(rng):
    hkv = rng.choice([1, 2, 3, 4])
    return hkv * rng.choice([1, 2, 4]), hkv


def _len(rng, lo, hi):
    if rng.random() < 0.5:
        base = rng.choice([128, 256, 384])
        return max(lo, min(hi, base + rng.choice([-1, 0, 1])))
    return rng.randint(lo, hi)


def _device_ok():
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"


def _grads(got, ref, what):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        if not np.any(r):
            assert float(g.float().abs().max()) <= 1e-3, f"{what} {name}"
            continue
        check_grad(g.cpu(), r, what=f"{what} {name}")


def _inputs(rng, B, Hq, Hkv, Sq, Sk, d, seed):
    q, k, v = W.prefill_inputs(B, Hq, Hkv, Sq, Sk, d, seed=seed, value_scale=0.5)
    do = W.grad_output(B, Hq, Sq, d, seed=seed, value_scale=0.5)
    return q, k, v, do


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_window_prefix(case):
    rng = random.Random(8000 + case)
    Hq, Hkv = _heads(rng)
    B = rng.randint(1, 2)
    Sq, Sk = _len(rng, 1, 600), _len(rng, 1, 600)
    d = rng.choice([64, 128])
    use_window = rng.random() < 0.6
    window = rng.randint(1, 400) if use_window else 0
    prefix = 0 if use_window else rng.randint(1, 400)
    scale = 1.0 / math.sqrt(d)
    q, k, v, do = _inputs(rng, B, Hq, Hkv, Sq, Sk, d, seed=8100 + case)
    qd, kd, vd, dod = (x.to(DEV) for x in (q, k, v, do))
    o, lse = attn_fwd_window(qd, kd, vd, scale, window=window, prefix=prefix)
    got = attn_bwd_window(qd, kd, vd, o, lse, dod, scale, window=window, prefix=prefix)
    torch.cuda.synchronize()
    _device_ok()
    what = f"B{B} Hq{Hq} Hkv{Hkv} Sq{Sq} Sk{Sk} d{d} w{window} p{prefix}"
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, True, scale, window=window, prefix=prefix)
    check(o.cpu(), o_ref, lse.cpu(), lse_ref, what=f"window fwd {what}")
    _grads(got, oracle_bwd(q, k, v, do, True, scale, window=window, prefix=prefix),
           f"window bwd {what}")


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_block_sparse(case):
    rng = random.Random(8200 + case)
    Hq, Hkv = _heads(rng)
    B = rng.randint(1, 2)
    Sq, Sk = _len(rng, 1, 600), _len(rng, 1, 600)
    d = rng.choice([64, 128])
    causal = rng.random() < 0.5
    per_head = rng.random() < 0.5
    density = rng.choice([0.25, 0.5, 0.9])
    scale = 1.0 / math.sqrt(d)
    q, k, v, do = _inputs(rng, B, Hq, Hkv, Sq, Sk, d, seed=8300 + case)
    g = torch.Generator().manual_seed(8400 + case)
    mask = (torch.rand(B, Hq if per_head else 1, -(-Sq // 128), -(-Sk // 128), generator=g)
            < density).to(torch.uint8)
    qd, kd, vd, dod, md = (x.to(DEV) for x in (q, k, v, do, mask))
    o, lse = attn_fwd_block_sparse(qd, kd, vd, md, causal, scale)
    got = attn_bwd_block_sparse(qd, kd, vd, o, lse, dod, md, causal, scale)
    torch.cuda.synchronize()
    _device_ok()
    what = f"B{B} Hq{Hq} Hkv{Hkv} Sq{Sq} Sk{Sk} d{d} c{causal} dens{density} ph{per_head}"
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, causal, scale, block_mask=mask.numpy())
    check(o.cpu(), o_ref, lse.cpu(), lse_ref, what=f"blocks fwd {what}")
    _grads(got, oracle_bwd(q, k, v, do, causal, scale, block_mask=mask.numpy()),
           f"blocks bwd {what}")


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_backward_padded(case):
    rng = random.Random(8500 + case)
    Hq, Hkv = _heads(rng)
    B = rng.randint(1, 3)
    Sq, Sk = _len(rng, 1, 600), _len(rng, 1, 600)
    d = rng.choice([64, 128])
    causal = rng.random() < 0.6
    scale = 1.0 / math.sqrt(d)
    q, k, v, do = _inputs(rng, B, Hq, Hkv, Sq, Sk, d, seed=8600 + case)
    k_lens = None
    if rng.random() < 0.5:
        k_lens = torch.tensor([rng.randint(0, Sk) for _ in range(B)], dtype=torch.int32)
    kl = None if k_lens is None else k_lens.to(DEV)
    qd, kd, vd, dod = (x.to(DEV) for x in (q, k, v, do))
    o, lse = attn_fwd_masked(qd, kd, vd, causal, scale, k_lens=kl)
    got = attn_bwd(qd, kd, vd, o, lse, dod, causal, scale, k_lens=kl)
    torch.cuda.synchronize()
    _device_ok()
    ref = oracle_bwd(q, k, v, do, causal, scale,
                     k_lens=None if k_lens is None else k_lens.numpy())
    _grads(got, ref, f"bwd B{B} Hq{Hq} Hkv{Hkv} Sq{Sq} Sk{Sk} d{d} c{causal} kl{k_lens}")


@pytest.mark.parametrize("case", range(N_CASES))
def test_fuzz_backward_ragged(case):
    rng = random.Random(8700 + case)
    Hq, Hkv = _heads(rng)
    B = rng.randint(1, 4)
    lens_q = [_len(rng, 0, 500) for _ in range(B)]
    lens_k = list(lens_q) if rng.random() < 0.5 else [_len(rng, 0, 500) for _ in range(B)]
    d = rng.choice([64, 128])
    causal = rng.random() < 0.6
    scale = 1.0 / math.sqrt(d)
    q, k, v, cu_q, cu_k = W.varlen_inputs(lens_q, lens_k, Hq, Hkv, d, seed=8800 + case,
                                         value_scale=0.5)
    do = W.randn_bf16(tuple(q.shape), 8900 + case, 0.5)
    max_q, max_k = max(max(lens_q), 1), max(max(lens_k), 1)
    qd, kd, vd, dod, cq, ck = (x.to(DEV) for x in (q, k, v, do, cu_q, cu_k))
    o, lse = attn_fwd_varlen(qd, kd, vd, cq, ck, max_q, causal, scale)
    got = attn_bwd_varlen(qd, kd, vd, o, lse, dod, cq, ck, max_q, max_k, causal, scale)
    torch.cuda.synchronize()
    _device_ok()
    ref = oracle_bwd_varlen(q, k, v, do, cu_q, cu_k, causal, scale)
    _grads(got, ref, f"ragged bwd q{lens_q} k{lens_k} Hq{Hq} Hkv{Hkv} d{d} c{causal}")
