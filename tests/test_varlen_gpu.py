"""GPU parity of attn_fwd_varlen (ragged batches through the C ABI) against the oracle.

"Attention Kernel", section "Paged 与 ragged KV": a ragged batch is described by
cumulative sequence lengths instead of padding; empty sequences and accesses
across sequence boundaries are part of the correctness contract.  Every case
draws seeded packed bf16 inputs on the host, runs the CUDA path on cuda:0 and
the float64 CPU oracle on the same bytes, and compares element by element
(``tests/parity.py`` states the bar) over every token that belongs to a
sequence.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_softmax_attention_fwd_b200 import (attn_fwd, attn_fwd_varlen, attn_get_device_error,
                                             workloads as W)

from parity import check

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _run(q, k, v, cu_q, cu_k, max_q, causal, scale):
    o, lse = attn_fwd_varlen(q.to(DEV), k.to(DEV), v.to(DEV), cu_q.to(DEV), cu_k.to(DEV), max_q,
                             causal, scale)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def _owned(cu_q, total_q):
    """Boolean mask of packed query tokens that belong to some sequence."""
    m = torch.zeros(total_q, dtype=torch.bool)
    for b in range(len(cu_q) - 1):
        m[int(cu_q[b]):int(cu_q[b + 1])] = True
    return m


def _case(lens_q, lens_k, Hq, Hkv, d, causal, seed, scale=None):
    q, k, v, cu_q, cu_k = W.varlen_inputs(lens_q, lens_k, Hq, Hkv, d, seed)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o, lse = _run(q, k, v, cu_q, cu_k, max(max(lens_q), 1), causal, scale)
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"
    o_ref, lse_ref = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, causal, scale)
    m = _owned(cu_q, q.shape[0])
    mn = m.numpy()
    return check(o[m], o_ref[mn], lse[:, m], lse_ref[:, mn],
                 what=f"varlen lens_q={lens_q} lens_k={lens_k} d{d} c{causal}")


MIXES = [
    # (lens_q, lens_k, Hq, Hkv, d, causal)
    ([1, 127, 128, 129, 255, 256, 257, 600], None, 4, 2, 128, True),
    ([300, 0, 17, 1000, 0, 5], None, 4, 1, 64, False),
    ([700, 333, 1], None, 8, 8, 64, True),
    ([513, 2048, 64], [1500, 2048, 300], 4, 2, 128, True),  # len_q != len_k: bottom-right diagonal
    ([256, 100], [0, 90], 2, 2, 128, True),                  # a sequence with no key at all
    ([4000], None, 8, 2, 128, True),                         # one long sequence
]


@pytest.mark.parametrize("case", MIXES, ids=[f"mix{i}" for i in range(len(MIXES))])
def test_ragged_mixes(case):
    lens_q, lens_k, Hq, Hkv, d, causal = case
    _case(lens_q, lens_k if lens_k is not None else lens_q, Hq, Hkv, d, causal, seed=61)


def test_worked_example_across_a_sequence_boundary():
    # "Attention Kernel", "Blockwise reference": scores [1, -inf, 3, -2, 0],
    # values arange(15) as 5 x 3.  The -inf key is realised as the first key of
    # the next sequence (value [3, 4, 5]); it sits in the same 128-key tile, is
    # read by the tile load and must get weight exactly 0.
    d = 64
    s = [1.0, 3.0, -2.0, 0.0, 5.0]
    vals = [[0, 1, 2], [6, 7, 8], [9, 10, 11], [12, 13, 14], [3, 4, 5]]
    q = torch.zeros(2, 1, d, dtype=torch.bfloat16)
    q[:, 0, 0] = 1.0
    k = torch.zeros(5, 1, d, dtype=torch.bfloat16)
    v = torch.zeros(5, 1, d, dtype=torch.bfloat16)
    for j in range(5):
        k[j, 0, 0] = s[j]
        v[j, 0, :3] = torch.tensor(vals[j], dtype=torch.bfloat16)
    cu_q = torch.tensor([0, 1, 2], dtype=torch.int32)
    cu_k = torch.tensor([0, 4, 5], dtype=torch.int32)
    o, lse = _run(q, k, v, cu_q, cu_k, 1, False, 1.0)
    np.testing.assert_allclose(o[0, 0, :3].double().numpy(),
                               [5.586297614919345, 6.586297614919345, 7.586297614919346],
                               atol=1e-2, rtol=0)
    assert torch.all(o[0, 0, 3:] == 0)
    assert abs(float(lse[0, 0]) - 3.1755153626167143) < 1e-3
    assert o[1, 0, :3].tolist() == [3.0, 4.0, 5.0] and abs(float(lse[0, 1]) - 5.0) < 1e-3


def test_equal_lengths_bitwise_equal_to_the_fixed_length_kernel():
    # the same tiles in the same order of arithmetic: identical bits
    B, Hq, Hkv, S, d = 3, 8, 2, 700, 128
    q, k, v = W.prefill_inputs(B, Hq, Hkv, S, S, d, seed=67)
    pk = lambda x: x.permute(0, 2, 1, 3).reshape(B * S, x.shape[1], d).contiguous()
    cu = W.cu_seqlens([S] * B)
    ov, lv = _run(pk(q), pk(k), pk(v), cu, cu, S, True, 1 / math.sqrt(d))
    of, lf = attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), True, 1 / math.sqrt(d))
    assert torch.equal(ov, pk(of.cpu()))
    assert torch.equal(lv, lf.cpu().permute(1, 0, 2).reshape(Hq, B * S))


def test_deterministic_bitwise():
    q, k, v, cu_q, cu_k = W.varlen_inputs([900, 40, 2100, 333], [900, 40, 2100, 333], 8, 2, 128,
                                          seed=71)
    a = _run(q, k, v, cu_q, cu_k, 2100, True, 0.088)
    b = _run(q, k, v, cu_q, cu_k, 2100, True, 0.088)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_bad_offsets_are_flagged_and_that_sequence_is_skipped():
    lens = [300, 200, 150]
    q, k, v, cu_q, cu_k = W.varlen_inputs(lens, lens, 2, 2, 64, seed=73)
    bad_k = cu_k.clone()
    bad_k[2] = int(bad_k[1]) - 1  # sequence 1's keys end before they start
    o = torch.full((q.shape[0], 2, 64), 7.0, dtype=torch.bfloat16, device=DEV)
    o, lse = attn_fwd_varlen(q.to(DEV), k.to(DEV), v.to(DEV), cu_q.to(DEV), bad_k.to(DEV), 300,
                             True, 0.125, out=o)
    torch.cuda.synchronize()
    st, flags = attn_get_device_error()
    assert flags & 0x4, "bad offsets must set ATTN_DEVERR_BAD_LENGTH"
    o, lse = o.cpu(), lse.cpu()
    assert torch.all(o[300:500] == 7.0)  # the bad sequence is left untouched
    # sequence 0 is unchanged; sequence 2 is now 150 queries over keys [299, 650)
    for (qa, qb), (ka, kb) in (((0, 300), (0, 300)), ((500, 650), (299, 650))):
        o_ref, lse_ref = oracle.attn_fwd_varlen(q[qa:qb], k[ka:kb], v[ka:kb], [0, qb - qa],
                                                [0, kb - ka], True, 0.125)
        check(o[qa:qb], o_ref, lse[:, qa:qb], lse_ref,
              what=f"valid sequence [{qa}, {qb}) next to a bad one")


def test_ragged_gqa_causal_sampled_rows():
    # the full ragged workload (16 sequences of 128..8192 tokens, GQA 32/8,
    # d = 128, causal) checked on seeded rows of every sequence
    c = W.CONFIGS["ragged_gqa_causal"]
    q, k, v, cu_q, cu_k, lens = W.varlen_config_inputs(c)
    o, lse = _run(q, k, v, cu_q, cu_k, int(lens.max()), True, c.scale)
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"
    g = torch.Generator().manual_seed(79)
    o_s, l_s, o_r, l_r = [], [], [], []
    for b in range(c.B):
        q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
        k0, k1 = int(cu_k[b]), int(cu_k[b + 1])
        n = q1 - q0
        qs = q[q0:q1].permute(1, 0, 2).unsqueeze(0).contiguous()
        ks = k[k0:k1].permute(1, 0, 2).unsqueeze(0).contiguous()
        vs = v[k0:k1].permute(1, 0, 2).unsqueeze(0).contiguous()
        rows = torch.randint(0, c.Hq * n, (24,), generator=g)
        rows = torch.unique(torch.cat([rows, torch.tensor([n - 1, c.Hq * n - 1])]))
        orow, lrow = oracle.attn_fwd(qs, ks, vs, True, c.scale, rows=rows)
        h, i = rows // n, rows % n
        o_s.append(o[q0 + i, h])
        l_s.append(lse[h, q0 + i])
        o_r.append(orow)
        l_r.append(lrow)
    check(torch.cat(o_s), np.concatenate(o_r), torch.cat(l_s), np.concatenate(l_r),
          what="ragged_gqa_causal sampled rows")
