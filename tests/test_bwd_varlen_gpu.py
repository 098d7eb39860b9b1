"""GPU parity of attn_bwd_varlen (the backward of a ragged, packed batch)
against the float64 backward oracle.

"Attention Kernel", section "Backward 与重计算": the backward must use the
forward's scale, mask and head mapping, and the boundaries of packed
sequences must agree with the forward's; section "Paged 与 ragged KV": each
sequence of a ragged batch is attended on its own.  The forward outputs come
from the CUDA ragged forward (the path a training step takes); gradients are
compared element by element over every token that belongs to a sequence.
"""
import math

import pytest
import torch

from oracle.attn_bwd import attn_bwd_varlen as oracle_bwd_varlen
from exact_softmax_attention_fwd_b200 import (attn_bwd, attn_bwd_varlen, attn_fwd_masked,
                                             attn_fwd_varlen, attn_get_device_error,
                                             workloads as W)

from parity import check_grad

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _owned(cu, total):
    m = torch.zeros(total, dtype=torch.bool)
    for b in range(len(cu) - 1):
        m[int(cu[b]):int(cu[b + 1])] = True
    return m


def _gpu(q, k, v, do, cu_q, cu_k, causal, scale, fill=None):
    lq = (cu_q[1:] - cu_q[:-1]).tolist()
    lk = (cu_k[1:] - cu_k[:-1]).tolist()
    mq, mk = max(max(lq), 1), max(max(lk), 1)
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), do.to(DEV)
    cqd, ckd = cu_q.to(DEV), cu_k.to(DEV)
    o, lse = attn_fwd_varlen(qd, kd, vd, cqd, ckd, mq, causal, scale)
    outs = [None, None, None]
    if fill is not None:  # tokens outside every sequence must keep their contents
        outs = [torch.full_like(qd, fill), torch.full_like(kd, fill), torch.full_like(vd, fill)]
    dq, dk, dv = attn_bwd_varlen(qd, kd, vd, o, lse, dod, cqd, ckd, mq, mk, causal, scale,
                                 dq=outs[0], dk=outs[1], dv=outs[2])
    torch.cuda.synchronize()
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"
    return dq.cpu(), dk.cpu(), dv.cpu()


MIXES = [
    # (lens_q, lens_k, Hq, Hkv, d, causal)
    ([1, 127, 128, 129, 255, 300], None, 4, 2, 128, True),
    ([300, 0, 17, 700, 5], None, 4, 1, 64, False),        # an empty sequence
    ([513, 1024, 64], [900, 1024, 300], 4, 2, 128, True),  # len_q != len_k: bottom-right
    ([200, 40, 90], [0, 300, 90], 8, 2, 128, True),       # a sequence with no key
    ([384, 129], [130, 640], 2, 2, 64, False),
]


@pytest.mark.parametrize("case", MIXES, ids=[f"mix{i}" for i in range(len(MIXES))])
def test_bwd_varlen_mixes(case):
    lens_q, lens_k, Hq, Hkv, d, causal = case
    lens_k = lens_q if lens_k is None else lens_k
    q, k, v, cu_q, cu_k = W.varlen_inputs(lens_q, lens_k, Hq, Hkv, d, seed=211)
    do = W.randn_bf16(tuple(q.shape), 211 * 16 + 7)
    scale = 1 / math.sqrt(d)
    dq, dk, dv = _gpu(q, k, v, do, cu_q, cu_k, causal, scale)
    rq, rk, rv = oracle_bwd_varlen(q, k, v, do, cu_q, cu_k, causal, scale)
    mq, mk = _owned(cu_q, q.shape[0]), _owned(cu_k, k.shape[0])
    check_grad(dq[mq], rq[mq.numpy()], what=f"dq {case}")
    check_grad(dk[mk], rk[mk.numpy()], what=f"dk {case}")
    check_grad(dv[mk], rv[mk.numpy()], what=f"dv {case}")


def test_bwd_varlen_leaves_foreign_tokens_alone():
    # packed tensors longer than the sequences: the rows after the last
    # sequence belong to nobody and must keep what the caller put there
    lens = [150, 77]
    q, k, v, cu_q, cu_k = W.varlen_inputs(lens + [40], lens + [60], 4, 2, 128, seed=213)
    cu_q, cu_k = cu_q[:3].clone(), cu_k[:3].clone()
    do = W.randn_bf16(tuple(q.shape), 213 * 16 + 7)
    dq, dk, dv = _gpu(q, k, v, do, cu_q, cu_k, True, 0.088, fill=3.0)
    assert torch.all(dq[227:] == 3.0) and torch.all(dk[227:] == 3.0) and torch.all(dv[227:] == 3.0)
    rq, rk, rv = oracle_bwd_varlen(q, k, v, do, cu_q, cu_k, True, 0.088)
    check_grad(dq[:227], rq[:227], what="dq")
    check_grad(dk[:227], rk[:227], what="dk")
    check_grad(dv[:227], rv[:227], what="dv")


def test_bwd_varlen_equal_lengths_bitwise_equal_to_fixed_length():
    """Equal lengths: the ragged call must give the fixed-length backward's bits
    (the same tiles in the same order; masked rows contribute exact zeros)."""
    B, Hq, Hkv, S, d = 3, 4, 2, 300, 128
    q, k, v = W.prefill_inputs(B, Hq, Hkv, S, S, d, seed=215)
    do = W.grad_output(B, Hq, S, d, seed=215)
    qd, kd, vd, dod = (x.to(DEV) for x in (q, k, v, do))
    o, lse = attn_fwd_masked(qd, kd, vd, True, 0.088)
    ref = attn_bwd(qd, kd, vd, o, lse, dod, True, 0.088)
    pk = lambda x: x.transpose(1, 2).reshape(-1, x.shape[1], d).contiguous()  # [B*S, H, d]
    cu = W.cu_seqlens([S] * B).to(DEV)
    lse_p = lse.permute(1, 0, 2).reshape(Hq, B * S).contiguous()
    got = attn_bwd_varlen(pk(qd), pk(kd), pk(vd), pk(o), lse_p, pk(dod), cu, cu, S, S, True, 0.088)
    torch.cuda.synchronize()
    for g, r in zip(got, ref):
        assert torch.equal(g, pk(r))


def test_bwd_varlen_bad_offsets_are_flagged():
    q, k, v, cu_q, cu_k = W.varlen_inputs([100, 50], [100, 50], 2, 2, 64, seed=217)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o, lse = attn_fwd_varlen(qd, kd, vd, cu_q.to(DEV), cu_k.to(DEV), 100, False, 0.125)
    bad = cu_q.clone()
    bad[1] = 500  # past total_q: sequence 0 and 1 are skipped
    attn_get_device_error()
    attn_bwd_varlen(qd, kd, vd, o, lse, qd, bad.to(DEV), cu_k.to(DEV), 100, 100, False, 0.125)
    st, flags = attn_get_device_error()
    assert st != 0 and flags & 0x4
