"""The decode entry point for callers that may not allocate device memory.

attn_decode_paged_noalloc keeps the split partials in the library's static
device scratch area instead of a caller workspace.  It must give the same
result as attn_decode_paged (same kernels) on consecutive calls that reuse the
area with stale contents, and must refuse problems larger than the area
without launching anything.  This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

from exact_softmax_attention_fwd_b200 import _binding as B
from exact_softmax_attention_fwd_b200 import workloads as W

from parity import check

DEV = "cuda:0"


def _to_dev(inp):
    return (inp.q.to(DEV), inp.k_cache.to(DEV), inp.v_cache.to(DEV), inp.block_table.to(DEV),
            inp.seq_lens.to(DEV))


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    c = W.CONFIGS["paged_decode"]
    problems = [
        (W.decode_config_inputs(c), c.scale),  # the full decode workload (about 17 MB of partials)
        (W.paged_inputs(torch.tensor([3000, 17, 0, 900], dtype=torch.int32), 32, 8, 128, 16,
                        seed=23), 0.09),
    ]
    for inp, scale in problems:  # the second call finds the first call's partials in the area
        q, kc, vc, tbl, lens = _to_dev(inp)
        o_ref, lse_ref = B.attn_decode_paged(q, kc, vc, tbl, lens, scale)
        o, lse = B.attn_decode_paged_noalloc(q, kc, vc, tbl, lens, scale)
        torch.cuda.synchronize()
        st, flags = B.attn_get_device_error()
        assert st == 0, f"device error flags {flags:#x}"
        check(o.cpu(), o_ref.cpu().double(), lse.cpu(), lse_ref.cpu().double(),
              what="no-alloc vs workspace entry point")
        # the same kernels in the same order: the results are the same bits
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


@pytest.mark.gpu
def test_noalloc_rejects_problems_beyond_the_scratch_area():
    # 64 x 64 heads x 4096 pages of 16 tokens needs ~270 MB of partials
    q = torch.zeros(64, 64, 128, dtype=torch.bfloat16, device=DEV)
    kc = torch.zeros(1, 16, 8, 128, dtype=torch.bfloat16, device=DEV)
    tbl = torch.zeros(64, 4096, dtype=torch.int32, device=DEV)
    lens = torch.zeros(64, dtype=torch.int32, device=DEV)
    need = B.attn_decode_workspace_size(64, 64, 4096, 16, 128)
    assert need > B.NOALLOC_SCRATCH_BYTES
    with pytest.raises(B.AttnError) as e:
        B.attn_decode_paged_noalloc(q, kc, kc, tbl, lens, 0.1)
    assert e.value.status == B.ATTN_ERR_WORKSPACE


def test_noalloc_size_check_happens_on_the_host():
    # no GPU needed: the size check comes before any CUDA call
    lib = B.load_library()
    fake = ctypes.c_void_p(0x100000)
    st = lib.attn_decode_paged_noalloc(fake, fake, fake, fake, fake, 16, 64, 64, 8, 128, 4096, 8,
                                       0.1, fake, None, None)
    assert st == B.ATTN_ERR_WORKSPACE
    assert lib.attn_decode_paged_noalloc(fake, fake, fake, fake, fake, 16, 0, 64, 8, 128, 4, 8,
                                         0.1, fake, None, None) == B.ATTN_ERR_INVALID_ARG
