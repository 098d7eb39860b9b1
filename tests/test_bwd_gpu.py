"""GPU parity of attn_bwd (the backward pass recomputing P from the saved LSE)
against the float64 backward oracle.

"Attention Kernel", section "Backward 与重计算": the backward recomputes the
local probabilities from Q, K, V, O and the log-sum-exp with the forward's
scale, mask and GQA mapping; accumulation must be race-free.  Inputs are
seeded bf16 on the host.  The forward outputs the CUDA backward consumes come
either from the oracle (O rounded to bf16, LSE to fp32), which isolates the
backward, or from the CUDA forward (the path a training step takes).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle.attn_bwd import attn_bwd as oracle_bwd
from exact_softmax_attention_fwd_b200 import (attn_bwd, attn_fwd_masked, attn_get_device_error,
                                             workloads as W)

from parity import check_grad

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _oracle_forward(q, k, v, causal, scale, k_lens=None):
    o, lse = oracle.attn_fwd(q, k, v, causal, scale, k_lens=None if k_lens is None else
                             k_lens.numpy())
    return (torch.from_numpy(o).to(torch.bfloat16), torch.from_numpy(lse).to(torch.float32))


def _gpu_bwd(q, k, v, o, lse, do, causal, scale, k_lens=None):
    kl = None if k_lens is None else k_lens.to(DEV)
    dq, dk, dv = attn_bwd(q.to(DEV), k.to(DEV), v.to(DEV), o.to(DEV), lse.to(DEV), do.to(DEV),
                          causal, scale, k_lens=kl)
    torch.cuda.synchronize()
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"
    return dq.cpu(), dk.cpu(), dv.cpu()


def _check_all(got, ref, what):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        check_grad(g, r, what=f"{what} {name}")


CASES = [
    # (B, Hq, Hkv, Sq, Sk, d, causal)
    (1, 2, 2, 300, 300, 128, True),
    (1, 4, 2, 333, 517, 128, True),    # Sq < Sk: the diagonal at the bottom right
    (2, 4, 1, 517, 333, 64, True),     # Sq > Sk: leading rows see no key
    (1, 2, 2, 256, 256, 64, False),
    (1, 3, 3, 200, 450, 128, False),
    (2, 8, 2, 384, 384, 128, True),    # GQA, 4 query heads per KV head
    (1, 2, 1, 130, 1000, 128, False),  # one ragged query tile, many key tiles
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_bwd_parity_oracle_forward(case):
    B, Hq, Hkv, Sq, Sk, d, causal = case
    q, k, v = W.prefill_inputs(B, Hq, Hkv, Sq, Sk, d, seed=171)
    do = W.grad_output(B, Hq, Sq, d, seed=171)
    scale = 1 / math.sqrt(d)
    o, lse = _oracle_forward(q, k, v, causal, scale)
    got = _gpu_bwd(q, k, v, o, lse, do, causal, scale)
    ref = oracle_bwd(q, k, v, do, causal, scale)
    _check_all(got, ref, f"bwd {case}")


def test_bwd_key_padding_and_empty_sequence():
    B, Hq, Hkv, S, d = 3, 4, 2, 400, 128
    q, k, v = W.prefill_inputs(B, Hq, Hkv, S, S, d, seed=172)
    do = W.grad_output(B, Hq, S, d, seed=172)
    k_lens = torch.tensor([400, 250, 0], dtype=torch.int32)
    scale = 1 / math.sqrt(d)
    for causal in (True, False):
        o, lse = _oracle_forward(q, k, v, causal, scale, k_lens)
        got = _gpu_bwd(q, k, v, o, lse, do, causal, scale, k_lens)
        ref = oracle_bwd(q, k, v, do, causal, scale, k_lens=k_lens.numpy())
        _check_all(got, ref, f"padding causal={causal}")
        # padded keys and the empty sequence get exact zeros
        assert not got[1][1, :, 250:].float().abs().sum() and not got[2][1, :, 250:].float().abs().sum()
        assert not got[0][2].float().abs().sum() and not got[1][2].float().abs().sum()


def test_bwd_chained_with_cuda_forward_mha_causal_2k():
    """The full mha_causal_2k workload (B=4, H=16, S=2048, d=128, causal), forward
    and backward both on the GPU, every gradient element against the oracle."""
    cfg = W.CONFIGS["mha_causal_2k"]
    q, k, v, _ = W.config_inputs(cfg)
    do = W.grad_output(cfg.B, cfg.Hq, cfg.S, cfg.d, seed=cfg.seed)
    scale = 1 / math.sqrt(cfg.d)
    o, lse = attn_fwd_masked(q.to(DEV), k.to(DEV), v.to(DEV), True, scale)
    got = _gpu_bwd(q, k, v, o.cpu(), lse.cpu(), do, True, scale)
    ref = oracle_bwd(q, k, v, do, True, scale)
    _check_all(got, ref, "mha_causal_2k")


def test_bwd_chained_with_cuda_forward_gqa_causal_8k_two_groups():
    """The gqa_causal_8k workload (B=2, Hq=32, Hkv=8, S=8192, d=128, causal, 4
    query heads per KV head), forward and backward on the GPU for the whole
    problem; every gradient element of two KV-head groups checked against the
    oracle: batch 0 with KV head 0 (query heads 0-3) and batch 1 with KV head 7
    (query heads 28-31).  Heads of different groups never interact, so the
    oracle on a group's slice gives that group's exact gradients, dK and dV
    summed over its four query heads."""
    cfg = W.CONFIGS["gqa_causal_8k"]
    q, k, v, _ = W.config_inputs(cfg)
    do = W.grad_output(cfg.B, cfg.Hq, cfg.S, cfg.d, seed=cfg.seed)
    scale = 1 / math.sqrt(cfg.d)
    o, lse = attn_fwd_masked(q.to(DEV), k.to(DEV), v.to(DEV), True, scale)
    dq, dk, dv = _gpu_bwd(q, k, v, o.cpu(), lse.cpu(), do, True, scale)
    g = cfg.Hq // cfg.Hkv
    for b, kvh in ((0, 0), (1, 7)):
        hs = slice(kvh * g, (kvh + 1) * g)
        sl = lambda x, h: x[b:b + 1, h].contiguous()
        ref = oracle_bwd(sl(q, hs), sl(k, slice(kvh, kvh + 1)), sl(v, slice(kvh, kvh + 1)),
                         sl(do, hs), True, scale)
        got = (sl(dq, hs), sl(dk, slice(kvh, kvh + 1)), sl(dv, slice(kvh, kvh + 1)))
        _check_all(got, ref, f"gqa_causal_8k batch {b} KV head {kvh}")


def test_bwd_is_deterministic():
    B, Hq, Hkv, S, d = 2, 8, 2, 700, 128
    q, k, v = [x.to(DEV) for x in W.prefill_inputs(B, Hq, Hkv, S, S, d, seed=173)]
    do = W.grad_output(B, Hq, S, d, seed=173).to(DEV)
    scale = 1 / math.sqrt(d)
    o, lse = attn_fwd_masked(q, k, v, True, scale)
    a = attn_bwd(q, k, v, o, lse, do, True, scale)
    b = attn_bwd(q, k, v, o, lse, do, True, scale)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))


def test_bwd_no_keys_gives_zero_dq():
    q = W.randn_bf16((1, 2, 100, 64), 174).to(DEV)
    k = torch.empty((1, 2, 0, 64), dtype=torch.bfloat16, device=DEV)
    o = torch.zeros_like(q)
    lse = torch.full((1, 2, 100), float("-inf"), device=DEV)
    dq = torch.full_like(q, 7.0)
    dq, dk, dv = attn_bwd(q, k, k, o, lse, q, True, 0.125, dq=dq)
    torch.cuda.synchronize()
    assert not dq.float().abs().sum().item() and dk.numel() == 0 and dv.numel() == 0


def test_bwd_bad_key_length_is_flagged_and_clamped():
    B, Hq, Hkv, S, d = 1, 2, 2, 256, 64
    q, k, v = W.prefill_inputs(B, Hq, Hkv, S, S, d, seed=175)
    do = W.grad_output(B, Hq, S, d, seed=175)
    scale = 1 / math.sqrt(d)
    o, lse = _oracle_forward(q, k, v, False, scale)
    dq, dk, dv = attn_bwd(q.to(DEV), k.to(DEV), v.to(DEV), o.to(DEV), lse.to(DEV), do.to(DEV),
                          False, scale, k_lens=torch.tensor([S + 9], dtype=torch.int32, device=DEV))
    st, flags = attn_get_device_error()
    assert st != 0 and flags & 0x4
    assert attn_get_device_error()[0] == 0  # reading clears the word
    ref = oracle_bwd(q, k, v, do, False, scale)  # clamped to S: no padding
    _check_all((dq.cpu(), dk.cpu(), dv.cpu()), ref, "clamped k_len")
