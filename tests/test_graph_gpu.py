"""CUDA-graph capture of the device entry points.

The C ABI allocates nothing per call and never synchronises a stream in a
launch, so its calls can be captured into a CUDA graph and replayed; the
decode merge kernel is launched as a programmatic dependent of the split
kernel, and the backward's dQ kernel as one of its dK/dV kernel, which a
graph has to keep as such.  Each case runs a call eagerly,
captures the same call (same buffers) into a graph, replays it and expects
the eager bits; then it rewrites the inputs in place (new values, shorter
lengths) and expects the replay to match an eager call on the new inputs.
"""
import math

import pytest
import torch

from exact_softmax_attention_fwd_b200 import (attn_bwd, attn_bwd_workspace_size,
                                             attn_decode_paged, attn_decode_paged_fp8,
                                             attn_decode_workspace_size, attn_fwd_masked,
                                             attn_fwd_varlen, attn_fwd_varlen_workspace_size,
                                             attn_get_device_error)
from exact_softmax_attention_fwd_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _device_ok():
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"


def _capture(fn):
    """Capture fn() on a side stream into a graph (after one eager warm-up)."""
    s = torch.cuda.Stream(device=DEV)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def _equal(a, b):
    return torch.equal(a.nan_to_num(posinf=1e30, neginf=-1e30),
                       b.nan_to_num(posinf=1e30, neginf=-1e30))


@pytest.mark.parametrize("fp8", [False, True])
def test_decode_replay_matches_eager(fp8):
    lens = torch.tensor([513, 1, 2048, 0, 777, 1500], dtype=torch.int32)
    Hq, Hkv, d, ps = 16, 4, 128, 16
    scale = 1.0 / math.sqrt(d)
    make = W.fp8_paged_inputs if fp8 else W.paged_inputs
    c = make(lens, Hq, Hkv, d, ps, seed=4242)
    q = c.q.to(DEV)
    kc, vc = c.k_cache.to(DEV), c.v_cache.to(DEV)
    tbl, sl = c.block_table.to(DEV), c.seq_lens.to(DEV)
    ks = c.k_scale.to(DEV) if fp8 else None
    vs = c.v_scale.to(DEV) if fp8 else None
    B = lens.numel()
    ws = torch.empty(attn_decode_workspace_size(B, Hq, tbl.shape[1], ps, d), dtype=torch.uint8,
                     device=DEV)
    o = torch.empty(B, Hq, d, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=DEV)

    def call(out=o, out_lse=lse):
        if fp8:
            attn_decode_paged_fp8(q, kc, vc, ks, vs, tbl, sl, scale, out=out, lse=out_lse,
                                  workspace=ws)
        else:
            attn_decode_paged(q, kc, vc, tbl, sl, scale, out=out, lse=out_lse, workspace=ws)

    o_ref, lse_ref = torch.empty_like(o), torch.empty_like(lse)
    call(o_ref, lse_ref)
    torch.cuda.synchronize()
    g = _capture(call)
    o.zero_()
    lse.zero_()
    g.replay()
    torch.cuda.synchronize()
    _device_ok()
    assert torch.equal(o, o_ref) and _equal(lse, lse_ref)

    # new query values and shorter lengths, written in place: the replay reads them
    q.copy_(torch.flip(q, dims=[0]))
    sl.copy_(torch.tensor([100, 0, 2048, 0, 16, 1499], dtype=torch.int32))
    g.replay()
    call(o_ref, lse_ref)
    torch.cuda.synchronize()
    _device_ok()
    assert torch.equal(o, o_ref) and _equal(lse, lse_ref)


def test_prefill_replay_matches_eager():
    B, Hq, Hkv, S, d = 2, 8, 2, 1000, 128
    scale = 1.0 / math.sqrt(d)
    q, k, v = (t.to(DEV) for t in W.prefill_inputs(B, Hq, Hkv, S, S, d, seed=99))
    kl = torch.tensor([1000, 617], dtype=torch.int32, device=DEV)
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, S, dtype=torch.float32, device=DEV)

    def call(out=o, out_lse=lse):
        attn_fwd_masked(q, k, v, True, scale, k_lens=kl, out=out, lse=out_lse)

    o_ref, lse_ref = torch.empty_like(o), torch.empty_like(lse)
    call(o_ref, lse_ref)
    g = _capture(call)
    o.zero_()
    g.replay()
    torch.cuda.synchronize()
    _device_ok()
    assert torch.equal(o, o_ref) and _equal(lse, lse_ref)
    k.mul_(0.5)
    kl.copy_(torch.tensor([333, 1000], dtype=torch.int32))
    g.replay()
    call(o_ref, lse_ref)
    torch.cuda.synchronize()
    _device_ok()
    assert torch.equal(o, o_ref) and _equal(lse, lse_ref)


def test_ragged_prefill_replay_matches_eager():
    lens = [300, 1, 1024, 700]
    Hq, Hkv, d = 8, 2, 128
    scale = 1.0 / math.sqrt(d)
    q, k, v, cu_q, cu_k = W.varlen_inputs(lens, lens, Hq, Hkv, d, seed=5150)
    q, k, v, cu_q, cu_k = (t.to(DEV) for t in (q, k, v, cu_q, cu_k))
    max_q = max(lens)
    o = torch.empty_like(q)
    lse = torch.empty(Hq, q.shape[0], dtype=torch.float32, device=DEV)
    ws = torch.empty(attn_fwd_varlen_workspace_size(len(lens), q.shape[0], max_q),
                     dtype=torch.uint8, device=DEV)

    def call(out=o, out_lse=lse):
        attn_fwd_varlen(q, k, v, cu_q, cu_k, max_q, True, scale, out=out, lse=out_lse,
                        workspace=ws)

    o_ref, lse_ref = torch.empty_like(o), torch.empty_like(lse)
    call(o_ref, lse_ref)
    g = _capture(call)
    o.zero_()
    g.replay()
    torch.cuda.synchronize()
    _device_ok()
    assert torch.equal(o, o_ref) and _equal(lse, lse_ref)


def test_backward_replay_matches_eager():
    B, Hq, Hkv, S, d = 2, 8, 2, 700, 128
    scale = 1.0 / math.sqrt(d)
    q, k, v = (t.to(DEV) for t in W.prefill_inputs(B, Hq, Hkv, S, S, d, seed=31, value_scale=0.5))
    d_o = W.grad_output(B, Hq, S, d, seed=32, value_scale=0.5).to(DEV)
    o, lse = attn_fwd_masked(q, k, v, True, scale)
    ws = torch.empty(attn_bwd_workspace_size(B, Hq, S), dtype=torch.uint8, device=DEV)
    grads = [torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)]

    def call(g=grads):
        attn_bwd(q, k, v, o, lse, d_o, True, scale, dq=g[0], dk=g[1], dv=g[2], workspace=ws)

    ref = [torch.empty_like(x) for x in grads]
    call(ref)
    graph = _capture(call)
    for x in grads:
        x.zero_()
    graph.replay()
    torch.cuda.synchronize()
    _device_ok()
    for x, y in zip(grads, ref):
        assert torch.equal(x, y)
    d_o.mul_(-2.0)
    graph.replay()
    call(ref)
    torch.cuda.synchronize()
    _device_ok()
    for x, y in zip(grads, ref):
        assert torch.equal(x, y)
