"""GPU parity of attn_fwd_paged (packed queries over a paged KV cache) against the oracle.

"Attention Kernel", section "Paged 与 ragged KV": key token t of a sequence lives
at offset t mod page_size of the physical page the block table gives for
logical page t / page_size; the last page is partial.  With a causal mask the
queries are the last len_q positions of their sequence (appending new tokens
to a cache that already holds them).  Inputs are seeded bf16 on the host; the
CUDA path runs on cuda:0, the float64 oracle on the same bytes.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_softmax_attention_fwd_b200 import (attn_decode_paged, attn_fwd_paged, attn_fwd_varlen,
                                             attn_get_device_error, workloads as W)

from parity import check

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _run(q, cu_q, c, max_q, causal, scale, table=None):
    tbl = c.block_table if table is None else table
    o, lse = attn_fwd_paged(q.to(DEV), c.k_cache.to(DEV), c.v_cache.to(DEV), tbl.to(DEV),
                            cu_q.to(DEV), c.seq_lens.to(DEV), max_q, causal, scale)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def _owned(cu_q, total):
    m = torch.zeros(total, dtype=torch.bool)
    for b in range(len(cu_q) - 1):
        m[int(cu_q[b]):int(cu_q[b + 1])] = True
    return m


MIXES = [
    # (lens_q, lens_k, Hq, Hkv, d, page_size, causal)
    ([100, 1, 300, 129], [700, 1, 300, 1000], 4, 2, 128, 16, True),   # append + full prefill + 1 token
    ([256, 0, 77], [2048, 50, 77], 8, 2, 64, 32, True),               # an empty query range
    ([200, 40], [1000, 0], 4, 4, 128, 64, True),                      # no cached key at all
    ([130, 600], [4000, 650], 8, 1, 128, 128, False),
    ([513], [3333], 8, 8, 64, 16, True),
]


@pytest.mark.parametrize("case", MIXES, ids=[f"mix{i}" for i in range(len(MIXES))])
def test_paged_prefill_mixes(case):
    lens_q, lens_k, Hq, Hkv, d, ps, causal = case
    q, cu_q, c = W.paged_prefill_inputs(lens_q, lens_k, Hq, Hkv, d, ps, seed=107)
    scale = 1 / math.sqrt(d)
    o, lse = _run(q, cu_q, c, max(max(lens_q), 1), causal, scale)
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"
    o_ref, lse_ref = oracle.attn_fwd_paged(q, c.k_cache, c.v_cache, c.block_table, cu_q,
                                           c.seq_lens, causal, scale)
    m = _owned(cu_q, q.shape[0])
    check(o[m], o_ref[m.numpy()], lse[:, m], lse_ref[:, m.numpy()], what=f"paged prefill {case}")


def test_contiguous_pages_bitwise_equal_to_ragged_kernel():
    lens_q, lens_k = [300, 1000, 45], [1200, 1000, 900]
    q, cu_q, c = W.paged_prefill_inputs(lens_q, lens_k, 8, 2, 128, 16, seed=109, contiguous=True)
    o, lse = _run(q, cu_q, c, 1000, True, 0.088)
    pk, pv = c.k_cache.reshape(-1, 2, 128), c.v_cache.reshape(-1, 2, 128)
    starts = [0]
    for n in lens_k:
        starts.append(starts[-1] + 16 * (-(-n // 16)))
    k = torch.cat([pk[starts[b]:starts[b] + lens_k[b]] for b in range(3)])
    v = torch.cat([pv[starts[b]:starts[b] + lens_k[b]] for b in range(3)])
    o2, l2 = attn_fwd_varlen(q.to(DEV), k.to(DEV), v.to(DEV), cu_q.to(DEV),
                             W.cu_seqlens(lens_k).to(DEV), 1000, True, 0.088)
    assert torch.equal(o, o2.cpu()) and torch.equal(lse, l2.cpu())


def test_single_token_queries_match_the_decode_kernel():
    lens_k = [1, 16, 17, 900, 4096]
    q, cu_q, c = W.paged_prefill_inputs([1] * 5, lens_k, 8, 2, 128, 16, seed=113)
    o, lse = _run(q, cu_q, c, 1, True, 0.1)
    od, ld = attn_decode_paged(q.to(DEV), c.k_cache.to(DEV), c.v_cache.to(DEV),
                               c.block_table.to(DEV), c.seq_lens.to(DEV), 0.1)
    torch.cuda.synchronize()
    check(o, od.cpu().double(), lse, ld.cpu().double().T, what="paged prefill vs decode kernel")


def test_bad_page_is_flagged_and_skipped():
    q, cu_q, c = W.paged_prefill_inputs([64, 64], [500, 500], 4, 2, 64, 16, seed=127)
    tbl = c.block_table.clone()
    tbl[0, 3] = c.k_cache.shape[0] + 5  # sequence 0, keys 48..63
    o, lse = _run(q, cu_q, c, 64, True, 0.125, table=tbl)
    st, flags = attn_get_device_error()
    assert flags & 0x2, "a page id outside the pool must set ATTN_DEVERR_BAD_PAGE"
    assert torch.isfinite(o.float()).all()
    # sequence 1 is untouched by the bad entry
    o_ref, lse_ref = oracle.attn_fwd_paged(q, c.k_cache, c.v_cache, c.block_table, cu_q,
                                           c.seq_lens, True, 0.125)
    check(o[64:], o_ref[64:], lse[:, 64:], lse_ref[:, 64:], what="sequence next to a bad page")


def test_paged_prefill_gqa_full():
    """Every token and head of the chunked-prefill workload (8 sequences x 1024
    new tokens over caches of 0..7168 tokens, pages of 16, Hq=32, Hkv=8)."""
    cfg = W.CONFIGS["paged_prefill_gqa"]
    q, cu_q, c, lq, lk = W.paged_prefill_config_inputs(cfg)
    o, lse = _run(q, cu_q, c, int(lq.max()), True, cfg.scale)
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"
    assert q.shape[0] == 8192
    o_ref, lse_ref = oracle.attn_fwd_paged(q, c.k_cache, c.v_cache, c.block_table, cu_q,
                                           c.seq_lens, True, cfg.scale)
    check(o, o_ref, lse, lse_ref, what="paged_prefill_gqa every token")
