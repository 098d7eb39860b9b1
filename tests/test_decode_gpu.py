"""GPU parity of attn_decode_paged (split-KV decode + merge) against the oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_softmax_attention_fwd_b200 import attn_decode_paged, attn_get_device_error
from exact_softmax_attention_fwd_b200 import workloads as W

from parity import check

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _run(inp, scale, workspace=None):
    o, lse = attn_decode_paged(inp.q.to(DEV), inp.k_cache.to(DEV), inp.v_cache.to(DEV),
                               inp.block_table.to(DEV), inp.seq_lens.to(DEV), scale,
                               workspace=workspace)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def _case(lens, Hq, Hkv, d, page_size, seed, scale=None, contiguous=False):
    inp = W.paged_inputs(torch.tensor(lens, dtype=torch.int32), Hq, Hkv, d, page_size, seed,
                         contiguous=contiguous, extra_pages=2)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o, lse = _run(inp, scale)
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"
    o_ref, lse_ref = oracle.decode_paged(inp.q, inp.k_cache, inp.v_cache, inp.block_table,
                                         inp.seq_lens, scale)
    return check(o, o_ref, lse, lse_ref, what=f"lens={lens[:4]} Hq{Hq} Hkv{Hkv} d{d} p{page_size}"), inp, o, lse


def test_paged_decode_config_full():
    c = W.CONFIGS["paged_decode"]
    inp = W.decode_config_inputs(c)
    o, lse = _run(inp, c.scale)
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"
    o_ref, lse_ref = oracle.decode_paged(inp.q, inp.k_cache, inp.v_cache, inp.block_table,
                                         inp.seq_lens, c.scale)
    check(o, o_ref, lse, lse_ref, what=c.name)


CASES = [
    # lens, Hq, Hkv, d, page_size
    ([1, 2, 15, 16, 17, 31, 32, 33], 32, 8, 128, 16),
    ([0, 5, 0, 600], 8, 2, 128, 16),              # empty sequences
    ([511, 512, 513, 1024, 1025, 1500], 4, 4, 128, 16),  # split boundaries (g = 1)
    ([700, 33, 4096], 16, 2, 128, 16),             # g = 8
    ([300, 1, 64], 8, 4, 64, 16),                  # d = 64, g = 2
    ([100, 257, 1000], 8, 2, 128, 32),             # page size 32
    ([129, 800], 6, 3, 64, 64),                    # page size 64, g = 2, odd heads
]


@pytest.mark.parametrize("case", CASES, ids=[str(c[1:]) + str(c[0][:3]) for c in CASES])
def test_decode_cases(case):
    lens, Hq, Hkv, d, ps = case
    _case(lens, Hq, Hkv, d, ps, seed=sum(lens) % 997 + d)


def test_contiguous_equals_permuted_pages():
    lens = [37, 600, 1111]
    _, a, oa, la = _case(lens, 8, 2, 128, 16, seed=5, contiguous=True)
    _, b, ob, lb = _case(lens, 8, 2, 128, 16, seed=5, contiguous=False)
    # same logical content, two physical placements: identical results
    kc = torch.empty_like(a.k_cache)
    vc = torch.empty_like(a.v_cache)
    for s, n in enumerate(lens):
        for p in range(-(-n // 16)):
            kc[int(b.block_table[s, p])] = a.k_cache[int(a.block_table[s, p])]
            vc[int(b.block_table[s, p])] = a.v_cache[int(a.block_table[s, p])]
    b2 = W.PagedInputs(a.q, kc, vc, b.block_table, b.seq_lens, 16)
    o2, l2 = _run(b2, 1 / math.sqrt(128))
    assert torch.equal(oa, o2) and torch.equal(la, l2)


def test_decode_deterministic():
    inp = W.paged_inputs(torch.tensor([3000, 17, 900], dtype=torch.int32), 32, 8, 128, 16, seed=7)
    o1, l1 = _run(inp, 0.088)
    o2, l2 = _run(inp, 0.088)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_decode_matches_prefill_row():
    # one decode query == the last row of a bottom-right causal prefill over the same keys
    from exact_softmax_attention_fwd_b200 import attn_fwd
    n, Hq, Hkv, d = 777, 8, 2, 128
    inp = W.paged_inputs(torch.tensor([n], dtype=torch.int32), Hq, Hkv, d, 16, seed=11,
                         contiguous=True)
    o, lse = _run(inp, 0.1)
    k = inp.k_cache.reshape(-1, Hkv, d)[:n].permute(1, 0, 2).unsqueeze(0).contiguous()
    v = inp.v_cache.reshape(-1, Hkv, d)[:n].permute(1, 0, 2).unsqueeze(0).contiguous()
    q = inp.q.reshape(1, Hq, 1, d).contiguous()
    o2, l2 = attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), True, 0.1)
    torch.cuda.synchronize()
    np.testing.assert_allclose(o[0].double().numpy(), o2.cpu()[0, :, 0].double().numpy(), atol=1e-2)
    np.testing.assert_allclose(lse[0].numpy(), l2.cpu()[0, :, 0].numpy(), atol=1e-3)


def test_worked_example_through_decode():
    # "Attention Kernel", section "Blockwise reference" example, as one decode
    # query over 4 visible tokens in a single (permuted) page.
    d = 64
    inp = W.paged_inputs(torch.tensor([4], dtype=torch.int32), 1, 1, d, 16, seed=13)
    q = torch.zeros(1, 1, d, dtype=torch.bfloat16)
    q[0, 0, 0] = 1.0
    page = int(inp.block_table[0, 0])
    s = [1.0, 3.0, -2.0, 0.0]
    vals = [[0, 1, 2], [6, 7, 8], [9, 10, 11], [12, 13, 14]]
    kc = inp.k_cache.clone()
    vc = inp.v_cache.clone()
    kc[page].zero_()
    vc[page].zero_()
    for t in range(4):
        kc[page, t, 0, 0] = s[t]
        vc[page, t, 0, :3] = torch.tensor(vals[t], dtype=torch.bfloat16)
    kc[page, 4, 0, 0] = 50.0  # slot past seq_len: must not be attended
    inp2 = W.PagedInputs(q, kc, vc, inp.block_table, inp.seq_lens, 16)
    o, lse = _run(inp2, 1.0)
    np.testing.assert_allclose(o[0, 0, :3].double().numpy(),
                               [5.586297614919345, 6.586297614919345, 7.586297614919346], atol=1e-2)
    assert abs(float(lse[0, 0]) - 3.1755153626167143) < 1e-3


def test_bad_page_id_flagged_not_faulting():
    inp = W.paged_inputs(torch.tensor([40, 40], dtype=torch.int32), 4, 2, 128, 16, seed=17)
    tbl = inp.block_table.clone()
    tbl[1, 1] = inp.num_pages + 1000  # outside the pool
    bad = W.PagedInputs(inp.q, inp.k_cache, inp.v_cache, tbl, inp.seq_lens, 16)
    attn_get_device_error()
    o, lse = _run(bad, 0.088)
    st, flags = attn_get_device_error()
    assert st != 0 and (flags & 0x2)
    assert torch.isfinite(o.float()).all()
    # the untouched sequence is still exact
    o_ref, lse_ref = oracle.decode_paged(inp.q, inp.k_cache, inp.v_cache, inp.block_table,
                                         inp.seq_lens, 0.088)
    check(o[0], o_ref[0], lse[0], lse_ref[0], what="unaffected sequence")
    st, flags = attn_get_device_error()
    assert st == 0


def test_slots_past_the_length_never_reach_the_result():
    """The last page of a sequence is partial; its unused slots (and a whole
    unused page) may hold anything, NaN included, without changing a bit."""
    inp = W.paged_inputs(torch.tensor([37, 500, 16], dtype=torch.int32), 8, 2, 128, 16, seed=19,
                         extra_pages=1)
    o1, l1 = _run(inp, 0.088)
    kc, vc = inp.k_cache.clone(), inp.v_cache.clone()
    for b, n in enumerate(inp.seq_lens.tolist()):
        last = int(inp.block_table[b, (n - 1) // 16])
        kc[last, n % 16 or 16:] = float("nan")
        vc[last, n % 16 or 16:] = float("nan")
    used = set(int(x) for x in inp.block_table.flatten().tolist() if x >= 0)
    unused = [pg for pg in range(inp.num_pages) if pg not in used]
    assert len(unused) == 1
    kc[unused[0]] = float("nan")  # the page no sequence references
    vc[unused[0]] = float("nan")
    o2, l2 = _run(W.PagedInputs(inp.q, kc, vc, inp.block_table, inp.seq_lens, 16), 0.088)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
