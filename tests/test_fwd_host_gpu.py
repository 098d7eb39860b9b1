"""GPU checks of attn_fwd_host, the prefill on host buffers with pipelined copies.

Its chunks are whole (sequence, KV head) pairs computed by the same prefill
kernel as attn_fwd_masked, so O and LSE must be bit-identical to that call on
the same bytes; one case also goes to the float64 oracle directly.  The cases
span several chunks, a ragged last chunk (B * Hkv not a multiple of the chunk
size), per-sequence key lengths, pageable memory, LSE omitted and Sk = 0.
"""
import math

import pytest
import torch

import oracle
from exact_softmax_attention_fwd_b200 import attn_fwd_host, attn_fwd_masked, attn_get_device_error
from exact_softmax_attention_fwd_b200 import workloads as W

from parity import check

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _device_reference(q, k, v, causal, scale, k_lens):
    kl = None if k_lens is None else k_lens.to(DEV)
    o, lse = attn_fwd_masked(q.to(DEV), k.to(DEV), v.to(DEV), causal, scale, k_lens=kl)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def _host_run(q, k, v, causal, scale, k_lens, pinned, return_lse=True):
    if pinned:
        q, k, v = q.pin_memory(), k.pin_memory(), v.pin_memory()
    o, lse = attn_fwd_host(q, k, v, causal, scale, k_lens=k_lens, return_lse=return_lse,
                           device=DEV)
    torch.cuda.synchronize()
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"
    return o, lse


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,d,causal,lens,pinned", [
    (3, 6, 3, 200, 333, 64, True, (333, 17, 0), True),    # 9 pairs: chunks of 2, last ragged
    (1, 8, 2, 1000, 1000, 128, False, None, False),       # 2 pairs, pageable memory
    (2, 32, 8, 2048, 2048, 128, True, None, True),        # 16 pairs: 8 chunks of 2
    (5, 4, 1, 130, 257, 128, True, (257, 1, 130, 200, 64), True),
])
def test_bit_identical_to_device_call(B, Hq, Hkv, Sq, Sk, d, causal, lens, pinned):
    q, k, v = W.prefill_inputs(B, Hq, Hkv, Sq, Sk, d, seed=B * 1000 + Sq)
    k_lens = None if lens is None else torch.tensor(lens, dtype=torch.int32)
    scale = 1.0 / math.sqrt(d)
    o, lse = _host_run(q, k, v, causal, scale, k_lens, pinned)
    o_ref, lse_ref = _device_reference(q, k, v, causal, scale, k_lens)
    assert o.device.type == "cpu" and lse.device.type == "cpu"
    assert torch.equal(o, o_ref)
    assert torch.equal(lse.nan_to_num(posinf=1e30, neginf=-1e30),
                       lse_ref.nan_to_num(posinf=1e30, neginf=-1e30))


def test_against_oracle_without_lse():
    B, Hq, Hkv, Sq, Sk, d = 2, 4, 2, 300, 300, 128
    q, k, v = W.prefill_inputs(B, Hq, Hkv, Sq, Sk, d, seed=77)
    k_lens = torch.tensor([300, 123], dtype=torch.int32)
    scale = 1.0 / math.sqrt(d)
    o, lse = _host_run(q, k, v, True, scale, k_lens, pinned=True, return_lse=False)
    assert lse is None
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, True, scale, k_lens=k_lens)
    check(o, o_ref, what="attn_fwd_host vs oracle")


def test_empty_keys():
    q, k, v = W.prefill_inputs(2, 4, 2, 64, 0, 128, seed=5)
    o, lse = _host_run(q, k, v, False, 0.1, None, pinned=True)
    assert torch.count_nonzero(o) == 0
    assert bool(torch.all(lse == float("-inf")))


def test_repeated_calls_reuse_one_workspace():
    """Back-to-back calls on one stream with one workspace: each result is its own."""
    B, Hq, Hkv, S, d = 2, 8, 4, 512, 128
    scale = 1.0 / math.sqrt(d)
    ws = torch.empty(1 << 26, dtype=torch.uint8, device=DEV)
    outs, refs = [], []
    for seed in (1, 2, 3):
        q, k, v = W.prefill_inputs(B, Hq, Hkv, S, S, d, seed=seed)
        q, k, v = q.pin_memory(), k.pin_memory(), v.pin_memory()
        outs.append(attn_fwd_host(q, k, v, True, scale, workspace=ws, device=DEV))
        refs.append(_device_reference(q, k, v, True, scale, None))
    torch.cuda.synchronize()
    for (o, lse), (o_ref, lse_ref) in zip(outs, refs):
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_concurrent_calls_from_two_host_threads():
    """Two host threads, each with its own stream and workspace, calling at once:
    the library's copy streams are shared, every result must still be its own."""
    import threading
    B, Hq, Hkv, S, d = 2, 8, 2, 384, 128
    scale = 1.0 / math.sqrt(d)
    cases = []
    for seed in (11, 12):
        q, k, v = W.prefill_inputs(B, Hq, Hkv, S, S, d, seed=seed)
        cases.append((q.pin_memory(), k.pin_memory(), v.pin_memory()))
    results = [None, None]
    errors = []

    def worker(t):
        try:
            stream = torch.cuda.Stream(device=DEV)
            ws = torch.empty(1 << 24, dtype=torch.uint8, device=DEV)
            outs = []
            for _ in range(3):
                outs.append(attn_fwd_host(*cases[t], True, scale, workspace=ws, device=DEV,
                                          stream=stream))
            stream.synchronize()
            results[t] = outs
        except Exception as e:  # surfaced below
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(t,)) for t in range(2)]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    assert not errors, errors
    for t in range(2):
        o_ref, lse_ref = _device_reference(*cases[t], True, scale, None)
        for o, lse in results[t]:
            assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
