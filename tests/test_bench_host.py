"""Host-side pieces of bench.py and the workload byte counts, on CPU.

* ncu traffic figures are keyed to a hash of one kernel family's own device
  sources: editing another family's header must not invalidate them, editing
  their own (or the shared primitives) must;
* a stale hash makes ``ncu_traffic`` report nothing rather than an old figure;
* the FP8 cache's algorithmic bytes: one byte per K and V element of the
  attended tokens plus the K and V scale of every page they touch;
* the visible (query, key) pairs the mask legs count their FLOPs over, against
  an element-by-element count of the same masks.
"""
import json
import os
import shutil

import pytest
import torch

import bench
from exact_softmax_attention_fwd_b200 import workloads as W

CSRC = os.path.join(bench.ROOT, "exact_softmax_attention_fwd_b200", "csrc")


@pytest.fixture
def fake_root(tmp_path, monkeypatch):
    """A copy of the sources and profiles under a temporary root."""
    dst = tmp_path / "exact_softmax_attention_fwd_b200" / "csrc"
    shutil.copytree(CSRC, dst, ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    shutil.copytree(os.path.join(bench.ROOT, "profiles"), tmp_path / "profiles")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path


def _touch(root, name):
    p = root / "exact_softmax_attention_fwd_b200" / "csrc" / name
    p.write_text(p.read_text() + "\n// edited\n")


def test_every_family_lists_existing_sources():
    for kernel, files in bench.KERNEL_SOURCES.items():
        for f in files:
            assert os.path.exists(os.path.join(CSRC, f)), (kernel, f)


def test_source_hash_is_per_kernel_family(fake_root):
    before = {k: bench.kernel_source_sha(k) for k in bench.KERNEL_SOURCES}
    _touch(fake_root, "bwd_sm100.cuh")
    after = {k: bench.kernel_source_sha(k) for k in bench.KERNEL_SOURCES}
    assert after["attn_bwd_dkdv_kernel"] != before["attn_bwd_dkdv_kernel"]
    assert after["attn_bwd_dq_kernel"] != before["attn_bwd_dq_kernel"]
    for k in ("attn_prefill_sm100_kernel", "attn_prefill_fp8_kernel",
              "attn_decode_split_tma_kernel", "attn_decode_split_tma_kernel_e4m3"):
        assert after[k] == before[k], k
    _touch(fake_root, "sm100_primitives.cuh")  # shared by every family
    again = {k: bench.kernel_source_sha(k) for k in bench.KERNEL_SOURCES}
    assert all(again[k] != after[k] for k in bench.KERNEL_SOURCES)


def test_stale_hash_hides_traffic(fake_root):
    with open(fake_root / "profiles" / "traffic.json") as f:
        t = json.load(f)
    kernel, cfgs = next(iter(t.items()))
    cfg = next(iter(cfgs))
    t[kernel][cfg]["source_sha"] = bench.kernel_source_sha(kernel)
    t[kernel][cfg]["dram_bytes_per_launch"] = 123.0
    with open(fake_root / "profiles" / "traffic.json", "w") as f:
        json.dump(t, f)
    assert bench.ncu_traffic(kernel, cfg) == 123.0
    for name in bench.KERNEL_SOURCES[kernel]:
        _touch(fake_root, name)
        break
    assert bench.ncu_traffic(kernel, cfg) is None
    assert bench.ncu_traffic(kernel, "no_such_workload") is None


def test_fp8_kv_bytes_formula():
    lens = torch.tensor([1, 16, 17, 0, 100], dtype=torch.int32)
    Hkv, d, ps = 8, 128, 16
    pages = 1 + 1 + 2 + 0 + 7
    assert W.fp8_kv_bytes(lens, Hkv, d, ps) == 134 * Hkv * d * 2 + pages * Hkv * 4 * 2
    # half the bf16 cache's K/V bytes, plus the scales
    assert W.fp8_kv_bytes(lens, Hkv, d, ps) - pages * Hkv * 8 == W.decode_kv_bytes(lens, Hkv, d) // 2


@pytest.mark.parametrize("S,window", [(1, 1), (300, 1), (300, 100), (300, 299), (300, 1000),
                                      (1024, 1024), (1030, 128)])
def test_window_visible_pairs(S, window):
    i = torch.arange(S)[:, None]
    j = torch.arange(S)[None, :]
    brute = int(((j <= i) & (j > i - window)).sum())
    assert bench.visible_pairs_window(S, window) == brute


@pytest.mark.parametrize("S,causal,density", [(1, True, 1.0), (128, True, 1.0), (300, True, 0.5),
                                               (300, False, 0.5), (513, True, 0.25),
                                               (640, False, 0.0)])
def test_block_mask_visible_pairs(S, causal, density):
    m = W.block_mask(2, 1, S, S, density, seed=17)
    i = torch.arange(S)[:, None]
    j = torch.arange(S)[None, :]
    vis = (j <= i) if causal else torch.ones(S, S, dtype=torch.bool)
    brute = 0
    for b in range(2):
        keep = m[b, 0].repeat_interleave(128, 0).repeat_interleave(128, 1)[:S, :S] > 0
        brute += int((vis & keep).sum())
    assert bench.visible_pairs_blocks(m, S, causal) == brute


def test_block_mask_generator_is_seeded_and_shaped():
    a = W.block_mask(2, 3, 300, 700, 0.4, seed=5)
    assert a.dtype == torch.uint8 and tuple(a.shape) == (2, 3, 3, 6)
    assert torch.equal(a, W.block_mask(2, 3, 300, 700, 0.4, seed=5))
    assert set(a.unique().tolist()) <= {0, 1}
