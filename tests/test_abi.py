"""CPU checks of the C ABI: the library loads, exports every declared symbol, and
rejects bad arguments on the host before touching CUDA (no compute calls)."""
import ctypes
import os
import re

import pytest

from exact_softmax_attention_fwd_b200 import _binding as B
from exact_softmax_attention_fwd_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(attn_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.load_library()


def test_header_declares_expected_entry_points():
    names = _declared_functions()
    for n in ("attn_fwd", "attn_fwd_masked", "attn_fwd_varlen", "attn_fwd_varlen_workspace_size",
              "attn_fwd_paged", "attn_fwd_window", "attn_fwd_block_sparse",
              "attn_decode_paged", "attn_decode_workspace_size", "attn_get_device_error",
              "attn_bwd", "attn_bwd_workspace_size", "attn_decode_paged_fp8", "attn_strerror"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), f"{name} declared in attn.h but not exported"
        assert name in B.SIGNATURES, f"{name} has no binding signature"


def test_strerror_covers_codes(lib):
    for code in range(0, 7):
        s = lib.attn_strerror(code).decode()
        assert s and s != "unknown status"
    assert lib.attn_strerror(99).decode() == "unknown status"


FAKE = 0x100000  # 16-byte aligned, never dereferenced: every call below fails validation


def _fwd(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, B_=1, Hq=2, Hkv=2, Sq=128, Sk=128, d=128,
         causal=0, scale=0.1, k_lens=None):
    return lib.attn_fwd_masked(q, k, v, o, lse, B_, Hq, Hkv, Sq, Sk, d, causal, scale, k_lens, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), B.ATTN_ERR_INVALID_ARG),
    (dict(o=None), B.ATTN_ERR_INVALID_ARG),
    (dict(B_=0), B.ATTN_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), B.ATTN_ERR_INVALID_ARG),
    (dict(Sq=0), B.ATTN_ERR_INVALID_ARG),
    (dict(Sk=-1), B.ATTN_ERR_INVALID_ARG),
    (dict(causal=2), B.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), B.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("inf")), B.ATTN_ERR_INVALID_ARG),
    (dict(d=96), B.ATTN_ERR_UNSUPPORTED),
    (dict(d=256), B.ATTN_ERR_UNSUPPORTED),
    (dict(q=FAKE + 8), B.ATTN_ERR_ALIGNMENT),
    (dict(v=FAKE + 2), B.ATTN_ERR_ALIGNMENT),
    (dict(lse=FAKE + 2), B.ATTN_ERR_ALIGNMENT),
    (dict(B_=70000), B.ATTN_ERR_INVALID_ARG),
])
def test_prefill_validation(lib, kw, status):
    assert _fwd(lib, **kw) == status


def test_prefill_plain_entry_validates_too(lib):
    assert lib.attn_fwd(None, FAKE, FAKE, FAKE, None, 1, 1, 1, 1, 1, 64, 0, 1.0, None) == \
        B.ATTN_ERR_INVALID_ARG


def _dec(lib, q=FAKE, kc=FAKE, vc=FAKE, tbl=FAKE, lens=FAKE, ps=16, B_=2, Hq=8, Hkv=2, d=128,
         maxp=4, npages=8, scale=0.1, o=FAKE, lse=None, ws=FAKE, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = lib.attn_decode_workspace_size(B_, Hq, maxp, ps, d) if B_ > 0 else 0
    return lib.attn_decode_paged(q, kc, vc, tbl, lens, ps, B_, Hq, Hkv, d, maxp, npages, scale, o,
                                 lse, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), B.ATTN_ERR_INVALID_ARG),
    (dict(tbl=None), B.ATTN_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), B.ATTN_ERR_INVALID_ARG),
    (dict(maxp=0), B.ATTN_ERR_INVALID_ARG),
    (dict(npages=0), B.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), B.ATTN_ERR_INVALID_ARG),
    (dict(ps=8), B.ATTN_ERR_UNSUPPORTED),
    (dict(ps=24), B.ATTN_ERR_UNSUPPORTED),
    (dict(d=80), B.ATTN_ERR_UNSUPPORTED),
    (dict(Hq=32, Hkv=2), B.ATTN_ERR_UNSUPPORTED),
    (dict(kc=FAKE + 4), B.ATTN_ERR_ALIGNMENT),
    (dict(ws=None), B.ATTN_ERR_WORKSPACE),
    (dict(ws_bytes=16), B.ATTN_ERR_WORKSPACE),
    (dict(ws=FAKE + 8), B.ATTN_ERR_ALIGNMENT),
    # 2^21 splits of 512 tokens x 2048 KV heads: more (split, KV head) CTAs than a grid row holds
    (dict(Hq=4096, Hkv=2048, maxp=1 << 22, ps=256), B.ATTN_ERR_INVALID_ARG),
])
def test_decode_validation(lib, kw, status):
    assert _dec(lib, **kw) == status


@pytest.mark.parametrize("window,prefix,status", [
    (-1, 0, B.ATTN_ERR_INVALID_ARG), (0, -1, B.ATTN_ERR_INVALID_ARG),
    (16, 16, B.ATTN_ERR_INVALID_ARG)])
def test_window_validation(lib, window, prefix, status):
    assert lib.attn_fwd_window(FAKE, FAKE, FAKE, FAKE, None, 1, 2, 2, 128, 128, 128, 0.1, None,
                               window, prefix, None) == status
    # the common checks still come first
    assert lib.attn_fwd_window(None, FAKE, FAKE, FAKE, None, 1, 2, 2, 128, 128, 128, 0.1, None,
                               16, 0, None) == B.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_window(FAKE, FAKE, FAKE, FAKE, None, 1, 2, 2, 128, 128, 96, 0.1, None,
                               16, 0, None) == B.ATTN_ERR_UNSUPPORTED


def test_block_sparse_validation(lib):
    args = (FAKE, FAKE, FAKE, FAKE, None, 1, 4, 2, 128, 128, 128, 1, 0.1, None)
    assert lib.attn_fwd_block_sparse(*args, None, 1, None) == B.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_block_sparse(*args, FAKE, 2, None) == B.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd_block_sparse(None, *args[1:], FAKE, 1, None) == B.ATTN_ERR_INVALID_ARG


def _var(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, cq=FAKE, ck=FAKE, B_=3, Hq=8, Hkv=2,
         tq=1000, tk=1000, maxq=512, d=128, causal=1, scale=0.1, ws=FAKE, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = lib.attn_fwd_varlen_workspace_size(B_, tq, maxq) if B_ > 0 else 0
    return lib.attn_fwd_varlen(q, k, v, o, lse, cq, ck, B_, Hq, Hkv, tq, tk, maxq, d, causal,
                               scale, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), B.ATTN_ERR_INVALID_ARG),
    (dict(cq=None), B.ATTN_ERR_INVALID_ARG),
    (dict(ck=None), B.ATTN_ERR_INVALID_ARG),
    (dict(k=None), B.ATTN_ERR_INVALID_ARG),
    (dict(B_=0), B.ATTN_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), B.ATTN_ERR_INVALID_ARG),
    (dict(tq=-1), B.ATTN_ERR_INVALID_ARG),
    (dict(tk=1 << 31), B.ATTN_ERR_INVALID_ARG),
    (dict(maxq=0), B.ATTN_ERR_INVALID_ARG),
    (dict(maxq=(1 << 21) + 1, ws_bytes=1 << 20), B.ATTN_ERR_INVALID_ARG),
    (dict(causal=3), B.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), B.ATTN_ERR_INVALID_ARG),
    (dict(d=96), B.ATTN_ERR_UNSUPPORTED),
    (dict(o=FAKE + 8), B.ATTN_ERR_ALIGNMENT),
    (dict(cq=FAKE + 2), B.ATTN_ERR_ALIGNMENT),
    (dict(ws=None), B.ATTN_ERR_WORKSPACE),
    (dict(ws_bytes=16), B.ATTN_ERR_WORKSPACE),
    (dict(ws=FAKE + 8), B.ATTN_ERR_ALIGNMENT),
])
def test_varlen_validation(lib, kw, status):
    assert _var(lib, **kw) == status


def test_varlen_empty_batch_launches_nothing(lib):
    # total_q = 0: nothing to compute, returns OK without touching a pointer
    assert _var(lib, tq=0) == B.ATTN_OK


def test_varlen_workspace_size_formula(lib):
    # one 16-byte header plus one int2 per possible (sequence, 256-row block)
    for B_, tq in ((1, 0), (16, 60592), (3, 1000)):
        assert lib.attn_fwd_varlen_workspace_size(B_, tq, 8192) == 16 + 8 * (tq // 256 + B_ + 1)
    assert lib.attn_fwd_varlen_workspace_size(0, 10, 10) == 0
    assert lib.attn_fwd_varlen_workspace_size(1, 10, 0) == 0


def _pp(lib, q=FAKE, kc=FAKE, vc=FAKE, tbl=FAKE, cq=FAKE, lk=FAKE, ps=16, B_=2, Hq=8, Hkv=2,
        tq=500, maxq=300, maxp=64, npages=100, d=128, causal=1, scale=0.1, o=FAKE, lse=None,
        ws=FAKE, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = lib.attn_fwd_varlen_workspace_size(B_, tq, maxq) if B_ > 0 else 0
    return lib.attn_fwd_paged(q, kc, vc, tbl, cq, lk, ps, B_, Hq, Hkv, tq, maxq, maxp, npages, d,
                              causal, scale, o, lse, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), B.ATTN_ERR_INVALID_ARG),
    (dict(tbl=None), B.ATTN_ERR_INVALID_ARG),
    (dict(lk=None), B.ATTN_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), B.ATTN_ERR_INVALID_ARG),
    (dict(maxp=0), B.ATTN_ERR_INVALID_ARG),
    (dict(npages=0), B.ATTN_ERR_INVALID_ARG),
    (dict(maxq=0), B.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("inf")), B.ATTN_ERR_INVALID_ARG),
    (dict(ps=8), B.ATTN_ERR_UNSUPPORTED),
    (dict(ps=48), B.ATTN_ERR_UNSUPPORTED),
    (dict(ps=256), B.ATTN_ERR_UNSUPPORTED),
    (dict(d=80), B.ATTN_ERR_UNSUPPORTED),
    (dict(kc=FAKE + 4), B.ATTN_ERR_ALIGNMENT),
    (dict(tbl=FAKE + 2), B.ATTN_ERR_ALIGNMENT),
    (dict(ws_bytes=8), B.ATTN_ERR_WORKSPACE),
])
def test_paged_prefill_validation(lib, kw, status):
    assert _pp(lib, **kw) == status


def test_workspace_size_formula(lib):
    split = lib.attn_split_tokens()
    assert split > 0 and split % 16 == 0
    B_, Hq, maxp, ps, d = 64, 32, 512, 16, 128
    n_split = -(-(maxp * ps) // split)
    parts = B_ * Hq * n_split
    got = lib.attn_decode_workspace_size(B_, Hq, maxp, ps, d)
    assert got >= parts * d * 4 + parts * 4
    assert got <= parts * d * 4 + parts * 4 + 256
    assert lib.attn_decode_workspace_size(0, 1, 1, 16, 128) == 0


def _dec8(lib, q=FAKE, kc=FAKE, vc=FAKE, ks=FAKE, vs=FAKE, tbl=FAKE, lens=FAKE, ps=16, B_=2, Hq=8,
          Hkv=2, d=128, maxp=4, npages=8, scale=0.1, o=FAKE, lse=None, ws=FAKE, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = lib.attn_decode_workspace_size(B_, Hq, maxp, ps, d) if B_ > 0 else 0
    return lib.attn_decode_paged_fp8(q, kc, vc, ks, vs, tbl, lens, ps, B_, Hq, Hkv, d, maxp,
                                     npages, scale, o, lse, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(ks=None), B.ATTN_ERR_INVALID_ARG),
    (dict(vs=None), B.ATTN_ERR_INVALID_ARG),
    (dict(q=None), B.ATTN_ERR_INVALID_ARG),
    (dict(kc=None), B.ATTN_ERR_INVALID_ARG),
    (dict(Hq=6, Hkv=4), B.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("inf")), B.ATTN_ERR_INVALID_ARG),
    (dict(ps=8), B.ATTN_ERR_UNSUPPORTED),
    (dict(d=96), B.ATTN_ERR_UNSUPPORTED),
    (dict(kc=FAKE + 8), B.ATTN_ERR_ALIGNMENT),
    (dict(vs=FAKE + 2), B.ATTN_ERR_ALIGNMENT),
    (dict(ks=FAKE + 1), B.ATTN_ERR_ALIGNMENT),
    (dict(ws_bytes=16), B.ATTN_ERR_WORKSPACE),
])
def test_decode_fp8_validation(lib, kw, status):
    assert _dec8(lib, **kw) == status


def _bwd(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, do=FAKE, dq=FAKE, dk=FAKE, dv=FAKE,
         B_=1, Hq=2, Hkv=1, Sq=200, Sk=300, d=128, causal=1, scale=0.1, k_lens=None, ws=FAKE,
         ws_bytes=1 << 20):
    return lib.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, B_, Hq, Hkv, Sq, Sk, d, causal, scale,
                        k_lens, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(o=None), B.ATTN_ERR_INVALID_ARG),
    (dict(lse=None), B.ATTN_ERR_INVALID_ARG),
    (dict(do=None), B.ATTN_ERR_INVALID_ARG),
    (dict(dq=None), B.ATTN_ERR_INVALID_ARG),
    (dict(dk=None), B.ATTN_ERR_INVALID_ARG),
    (dict(ws=None), B.ATTN_ERR_INVALID_ARG),
    (dict(q=None), B.ATTN_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), B.ATTN_ERR_INVALID_ARG),
    (dict(Sq=0), B.ATTN_ERR_INVALID_ARG),
    (dict(causal=3), B.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), B.ATTN_ERR_INVALID_ARG),
    (dict(d=80), B.ATTN_ERR_UNSUPPORTED),
    (dict(do=FAKE + 8), B.ATTN_ERR_ALIGNMENT),
    (dict(dv=FAKE + 2), B.ATTN_ERR_ALIGNMENT),
    (dict(o=FAKE + 4), B.ATTN_ERR_ALIGNMENT),
    (dict(ws=FAKE + 8), B.ATTN_ERR_ALIGNMENT),
    (dict(lse=FAKE + 2), B.ATTN_ERR_ALIGNMENT),
    (dict(ws_bytes=2 * 2 * 256 * 4 - 1), B.ATTN_ERR_WORKSPACE),
])
def test_bwd_validation(lib, kw, status):
    assert _bwd(lib, **kw) == status


def test_bwd_workspace_size_formula(lib):
    # two fp32 statistics per query row, rows padded to whole 128-row tiles
    assert lib.attn_bwd_workspace_size(1, 2, 200) == 2 * 2 * 256 * 4
    assert lib.attn_bwd_workspace_size(4, 16, 2048) == 2 * 64 * 2048 * 4
    assert lib.attn_bwd_workspace_size(0, 1, 1) == 0
    assert lib.attn_bwd_workspace_size(1, 1, 0) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 16, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        B.attn_fwd(q, q, q, False, 0.1)


def test_binding_checks_caller_output_buffers():
    import torch
    cpu = torch.device("cpu")
    good = torch.empty((2, 3, 4), dtype=torch.bfloat16)
    assert B._out(good, (2, 3, 4), torch.bfloat16, cpu, "out") is good
    fresh = B._out(None, (2, 3), torch.float32, cpu, "lse")
    assert tuple(fresh.shape) == (2, 3) and fresh.dtype == torch.float32
    for bad in (torch.empty((2, 3, 5), dtype=torch.bfloat16),      # too small a row
                torch.empty((2, 3, 4), dtype=torch.float16),       # wrong dtype
                torch.empty((2, 4, 3), dtype=torch.bfloat16).transpose(1, 2)):  # not contiguous
        with pytest.raises(ValueError):
            B._out(bad, (2, 3, 4), torch.bfloat16, cpu, "out")


@pytest.mark.parametrize("entry", ["attn_decode_paged", "attn_decode_paged_noalloc"])
def test_decode_binding_refuses_non_bf16_q_and_caches(entry):
    # an E4M3 cache (uint8, the FP8 decode's layout) or an fp16 q would be read
    # as bf16 bytes; the binding rejects them before any CUDA call
    import torch
    fn = getattr(B, entry)
    q = torch.zeros(2, 4, 128, dtype=torch.bfloat16)
    cache = torch.zeros(3, 16, 2, 128, dtype=torch.bfloat16)
    cache8 = torch.zeros(3, 16, 2, 128, dtype=torch.uint8)
    tbl = torch.zeros(2, 2, dtype=torch.int32)
    lens = torch.ones(2, dtype=torch.int32)
    for args in ((q, cache8, cache8), (q, cache, cache8), (q.half(), cache, cache),
                 (q.float(), cache, cache)):
        with pytest.raises(ValueError, match="bfloat16"):
            fn(*args, tbl, lens, 0.1)


def test_fp8_decode_binding_refuses_non_bf16_q():
    import torch
    q = torch.zeros(2, 4, 128, dtype=torch.float16)
    c8 = torch.zeros(3, 16, 2, 128, dtype=torch.uint8)
    sc = torch.ones(3, 2, dtype=torch.float32)
    with pytest.raises(ValueError, match="bfloat16"):
        B.attn_decode_paged_fp8(q, c8, c8, sc, sc, torch.zeros(2, 2, dtype=torch.int32),
                                torch.ones(2, dtype=torch.int32), 0.1)


def test_noalloc_scratch_size_matches_the_header():
    text = open(HEADER).read()
    m = re.search(r"#define\s+ATTN_NOALLOC_SCRATCH_BYTES\s+\(?([^\n/]+?)\)?\s*(?://.*)?$", text,
                  flags=re.M)
    assert m, "ATTN_NOALLOC_SCRATCH_BYTES not found in attn.h"
    expr = m.group(1).replace("u", "").replace("U", "").replace("ll", "").replace("LL", "")
    assert eval(expr, {}, {}) == B.NOALLOC_SCRATCH_BYTES


def _bwd_varlen(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, do=FAKE, dq=FAKE, dk=FAKE, dv=FAKE,
                cu_q=FAKE, cu_k=FAKE, B_=2, Hq=2, Hkv=1, total_q=300, total_k=400, max_q=200,
                max_k=250, d=128, causal=1, scale=0.1, ws=FAKE, ws_bytes=1 << 20):
    return lib.attn_bwd_varlen(q, k, v, o, lse, do, dq, dk, dv, cu_q, cu_k, B_, Hq, Hkv, total_q,
                               total_k, max_q, max_k, d, causal, scale, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), B.ATTN_ERR_INVALID_ARG),
    (dict(cu_q=None), B.ATTN_ERR_INVALID_ARG),
    (dict(cu_k=None), B.ATTN_ERR_INVALID_ARG),
    (dict(dk=None), B.ATTN_ERR_INVALID_ARG),
    (dict(B_=0), B.ATTN_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), B.ATTN_ERR_INVALID_ARG),
    (dict(total_q=-1), B.ATTN_ERR_INVALID_ARG),
    (dict(max_q=0), B.ATTN_ERR_INVALID_ARG),
    (dict(max_k=0), B.ATTN_ERR_INVALID_ARG),
    (dict(causal=2), B.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("inf")), B.ATTN_ERR_INVALID_ARG),
    (dict(d=96), B.ATTN_ERR_UNSUPPORTED),
    (dict(q=FAKE + 8), B.ATTN_ERR_ALIGNMENT),
    (dict(cu_q=FAKE + 2), B.ATTN_ERR_ALIGNMENT),
    (dict(lse=FAKE + 1), B.ATTN_ERR_ALIGNMENT),
    (dict(ws=FAKE + 4), B.ATTN_ERR_ALIGNMENT),
    (dict(ws_bytes=2 * 2 * 2 * 256 * 4 - 1), B.ATTN_ERR_WORKSPACE),
])
def test_bwd_varlen_validation(lib, kw, status):
    assert _bwd_varlen(lib, **kw) == status


def test_bwd_varlen_workspace_size_formula(lib):
    # two fp32 statistics per query row; every sequence padded to max_seqlen_q in 128-row tiles
    assert lib.attn_bwd_varlen_workspace_size(2, 2, 200) == 2 * 2 * 2 * 256 * 4
    assert lib.attn_bwd_varlen_workspace_size(16, 32, 8192) == 2 * 16 * 32 * 8192 * 4
    assert lib.attn_bwd_varlen_workspace_size(0, 1, 1) == 0


def _fwd_fp8(lib, q=FAKE, k=FAKE, v=FAKE, qs=FAKE, ks=FAKE, vs=FAKE, o=FAKE, lse=None, B_=1,
             Hq=2, Hkv=2, Sq=128, Sk=128, d=128, causal=0, scale=0.1, k_lens=None):
    return lib.attn_fwd_fp8(q, k, v, qs, ks, vs, o, lse, B_, Hq, Hkv, Sq, Sk, d, causal, scale,
                            k_lens, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), B.ATTN_ERR_INVALID_ARG),
    (dict(qs=None), B.ATTN_ERR_INVALID_ARG),
    (dict(vs=None), B.ATTN_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), B.ATTN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), B.ATTN_ERR_INVALID_ARG),
    (dict(d=64), B.ATTN_ERR_UNSUPPORTED),
    (dict(k=FAKE + 8), B.ATTN_ERR_ALIGNMENT),
    (dict(ks=FAKE + 2), B.ATTN_ERR_ALIGNMENT),
])
def test_fwd_fp8_validation(lib, kw, status):
    assert _fwd_fp8(lib, **kw) == status


def test_fp8_prefill_binding_checks_codes_and_scales():
    import torch
    q8 = torch.zeros(1, 2, 130, 128, dtype=torch.uint8)
    qs = torch.ones(1, 2, 2, dtype=torch.float32)
    with pytest.raises(ValueError, match="uint8"):
        B.attn_fwd_fp8(q8.float(), q8, q8, qs, qs, qs, True, 0.1)
    with pytest.raises(ValueError, match="block scales"):  # one per 128-row block: [1, 2, 2]
        B.attn_fwd_fp8(q8, q8, q8, qs[:, :, :1].contiguous(), qs, qs, True, 0.1)


def test_bwd_masked_entry_validation(lib):
    F_ = FAKE
    # window and prefix together, or negative: rejected before any CUDA call
    args = [F_] * 9 + [1, 2, 1, 200, 200, 128, 0.1, None]
    assert lib.attn_bwd_window(*args, 16, 16, F_, 1 << 20, None) == B.ATTN_ERR_INVALID_ARG
    assert lib.attn_bwd_window(*args, -1, 0, F_, 1 << 20, None) == B.ATTN_ERR_INVALID_ARG
    assert lib.attn_bwd_window(*args[:14], 80, 0.1, None, 16, 0, F_, 1 << 20,
                               None) == B.ATTN_ERR_UNSUPPORTED
    bargs = [F_] * 9 + [1, 2, 1, 200, 200, 128, 1, 0.1, None]
    assert lib.attn_bwd_block_sparse(*bargs, None, 1, F_, 1 << 20, None) == B.ATTN_ERR_INVALID_ARG
    assert lib.attn_bwd_block_sparse(*bargs, F_, 3, F_, 1 << 20, None) == B.ATTN_ERR_INVALID_ARG
    assert lib.attn_bwd_block_sparse(*bargs, F_, 1, F_, 16, None) == B.ATTN_ERR_WORKSPACE


def test_paged_fp8_validation(lib):
    F_ = FAKE
    base = dict(q=F_, k=F_, v=F_, ks=F_, vs=F_, tbl=F_, cuq=F_, lens=F_, ps=16, B_=2, Hq=4, Hkv=2,
                tq=100, mq=64, mp=8, np_=16, d=128, causal=1, scale=0.1, o=F_, lse=None, ws=F_,
                wsb=1 << 30)

    def call(**kw):
        a = dict(base, **kw)
        return lib.attn_fwd_paged_fp8(a["q"], a["k"], a["v"], a["ks"], a["vs"], a["tbl"], a["cuq"],
                                      a["lens"], a["ps"], a["B_"], a["Hq"], a["Hkv"], a["tq"],
                                      a["mq"], a["mp"], a["np_"], a["d"], a["causal"], a["scale"],
                                      a["o"], a["lse"], a["ws"], a["wsb"], None)
    assert call(ks=None) == B.ATTN_ERR_INVALID_ARG
    assert call(vs=None) == B.ATTN_ERR_INVALID_ARG
    assert call(ps=24) == B.ATTN_ERR_UNSUPPORTED
    assert call(d=96) == B.ATTN_ERR_UNSUPPORTED
    assert call(ks=F_ + 2) == B.ATTN_ERR_ALIGNMENT
    assert call(wsb=1024) == B.ATTN_ERR_WORKSPACE
    need = lib.attn_fwd_paged_fp8_workspace_size(2, 100, 64, 8, 16, 2, 128)
    # unit list + table + two bf16 pools of B * max_pages pages
    assert need >= 2 * 2 * 8 * 16 * 2 * 128 * 2
    assert lib.attn_fwd_paged_fp8_workspace_size(0, 100, 64, 8, 16, 2, 128) == 0


def test_fwd_host_validation(lib):
    F_ = FAKE

    def call(q=F_, lens=None, ws=F_, wsb=1 << 40, d=128, Hq=4, Hkv=2, Sk=300):
        return lib.attn_fwd_host(q, F_, F_, F_, None, 2, Hq, Hkv, 200, Sk, d, 1, 0.1, lens, ws, wsb,
                                 None)
    assert call(q=None) == B.ATTN_ERR_INVALID_ARG
    assert call(Hq=3) == B.ATTN_ERR_INVALID_ARG
    assert call(d=96) == B.ATTN_ERR_UNSUPPORTED
    assert call(ws=None) == B.ATTN_ERR_WORKSPACE
    assert call(wsb=1024) == B.ATTN_ERR_WORKSPACE
    assert call(ws=F_ + 4) == B.ATTN_ERR_ALIGNMENT
    # host key lengths are checked on the host, before any copy
    for bad in ((300, 301), (-1, 5)):
        lens = (ctypes.c_int32 * 2)(*bad)
        assert call(lens=ctypes.cast(lens, ctypes.c_void_p)) == B.ATTN_ERR_INVALID_ARG


def test_fwd_host_workspace_size_formula(lib):
    def up(x):
        return (x + 255) // 256 * 256
    for (B_, Hq, Hkv, Sq, Sk, d) in ((1, 32, 8, 32768, 32768, 128), (3, 6, 3, 200, 333, 64),
                                     (2, 4, 4, 1, 0, 128)):
        pairs, G = B_ * Hkv, Hq // Hkv
        ppc = (pairs + 7) // 8  # about eight chunks of whole (sequence, KV head) pairs
        qb, kvb, lb = ppc * G * Sq * d * 2, ppc * Sk * d * 2, ppc * G * Sq * 4
        want = 2 * (2 * up(qb) + 2 * up(kvb) + up(lb)) + up(pairs * 4)
        assert lib.attn_fwd_host_workspace_size(B_, Hq, Hkv, Sq, Sk, d) == want
    assert lib.attn_fwd_host_workspace_size(1, 3, 2, 128, 128, 128) == 0
    assert lib.attn_fwd_host_workspace_size(1, 4, 2, 128, 128, 96) == 0


def test_fwd_host_binding_refuses_device_tensors():
    import torch
    q = torch.zeros(1, 2, 8, 128, dtype=torch.bfloat16, device="meta")
    with pytest.raises(ValueError, match="host"):
        B.attn_fwd_host(q, q, q, True, 0.1)
