"""GPU parity of attn_fwd / attn_fwd_masked (through the C ABI) against the oracle.

Every case draws seeded bf16 inputs on the host, runs the CUDA path on cuda:0
and the float64 CPU oracle on the same bytes, and compares element by element
(``tests/parity.py`` states the bar).  The workloads up to 8k (and its padded
variant) are checked on every element; the 32k workload on its 512 seeded
(head, query row) pairs, which the oracle computes one by one.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from exact_softmax_attention_fwd_b200 import attn_fwd, attn_fwd_masked, attn_get_device_error
from exact_softmax_attention_fwd_b200 import workloads as W

from parity import check

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _run(q, k, v, causal, scale, k_lens=None):
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    kl = None if k_lens is None else k_lens.to(DEV)
    o, lse = attn_fwd_masked(qd, kd, vd, causal, scale, k_lens=kl)
    torch.cuda.synchronize()
    st, flags = attn_get_device_error()
    assert st == 0, f"device error flags {flags:#x}"
    return o.cpu(), lse.cpu()


def _full_case(B, Hq, Hkv, Sq, Sk, d, causal, seed, scale=None, k_lens=None, value_scale=1.0):
    q, k, v = W.prefill_inputs(B, Hq, Hkv, Sq, Sk, d, seed, value_scale)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    o, lse = _run(q, k, v, causal, scale, k_lens)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, causal, scale, k_lens=k_lens)
    return check(o, o_ref, lse, lse_ref, what=f"B{B} Hq{Hq} Hkv{Hkv} Sq{Sq} Sk{Sk} d{d} c{causal}")


def _sampled_case(cfg, n_rows, seed, extra_rows=None):
    q, k, v, k_lens = W.config_inputs(cfg)
    o, lse = _run(q, k, v, cfg.causal, cfg.scale, k_lens)
    rows = W.sample_rows(cfg.B, cfg.Hq, cfg.S, n_rows, seed)
    if extra_rows is not None:
        rows = torch.unique(torch.cat([rows, extra_rows]))
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, cfg.causal, cfg.scale, k_lens=k_lens, rows=rows)
    d = cfg.d
    o_s = o.reshape(-1, d)[rows]
    lse_s = lse.reshape(-1)[rows]
    return check(o_s, o_ref, lse_s, lse_ref, what=cfg.name), o, lse, k_lens


# ----------------------------------------------------------------- the named workloads


def test_tiny_mha_full():
    c = W.CONFIGS["tiny_mha"]
    _full_case(c.B, c.Hq, c.Hkv, c.S, c.S, c.d, c.causal, c.seed)


def test_mha_causal_2k_full():
    c = W.CONFIGS["mha_causal_2k"]
    q, k, v, _ = W.config_inputs(c)
    o, lse = _run(q, k, v, c.causal, c.scale)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, c.causal, c.scale)
    check(o, o_ref, lse, lse_ref, what=c.name)


def test_gqa_causal_8k_full():
    """Every element of the 8k GQA workload (B=2, Hq=32, Hkv=8, S=8192) against
    the oracle: 524,288 rows, about 1.1e12 float64 multiply-adds on the host."""
    c = W.CONFIGS["gqa_causal_8k"]
    q, k, v, _ = W.config_inputs(c)
    o, lse = _run(q, k, v, c.causal, c.scale)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, c.causal, c.scale)
    check(o, o_ref, lse, lse_ref, what=c.name)


def test_gqa_causal_8k_padded_full():
    """Every element of the padded 8k workload (keys past k_len[b] masked, with
    bottom-right causal alignment, so rows i < S - k_len[b] of every head see no
    key): compared with the oracle everywhere, and the fully masked rows of all
    heads exactly zero with LSE = -inf."""
    c = W.CONFIGS["gqa_causal_8k_padded"]
    B, S = c.B, c.S
    q, k, v, kl = W.config_inputs(c)
    assert kl is not None and int((S - kl).max()) > 0
    o, lse = _run(q, k, v, c.causal, c.scale, kl)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, c.causal, c.scale, k_lens=kl)
    stats = check(o, o_ref, lse, lse_ref, what=c.name)
    for b in range(B):
        n_empty = S - int(kl[b])
        assert torch.all(o[b, :, :n_empty] == 0)
        assert torch.all(torch.isneginf(lse[b, :, :n_empty]))
        assert torch.all(torch.isfinite(lse[b, :, n_empty:]))
    assert stats["empty_rows"] == c.Hq * int((S - kl).sum())


def test_gqa_causal_32k_512_pairs():
    c = W.CONFIGS["gqa_causal_32k"]
    _sampled_case(c, 512, seed=41)


# ----------------------------------------------------------------- edge cases


EDGE_CASES = [
    # B, Hq, Hkv, Sq, Sk, d, causal
    (1, 1, 1, 1, 1, 64, False),       # S_q = S_k = 1
    (1, 2, 1, 1, 300, 128, True),     # decode-like row: bottom-right causal sees every key
    (2, 4, 2, 200, 200, 128, True),   # ragged single tile pair
    (1, 2, 2, 333, 333, 64, True),    # ragged, several tiles
    (1, 2, 2, 333, 129, 64, False),   # Sk just past one tile
    (1, 4, 1, 129, 517, 128, True),   # Sq < Sk, bottom-right causal, GQA 4
    (2, 2, 2, 300, 100, 128, True),   # Sq > Sk: leading rows fully masked
    (1, 8, 1, 640, 640, 128, False),  # MQA, several KV tiles, non-causal
    (1, 3, 3, 520, 777, 64, False),   # odd head count, ragged
    (1, 2, 2, 1024, 1024, 128, True),
]


@pytest.mark.parametrize("case", EDGE_CASES, ids=[str(c) for c in EDGE_CASES])
def test_edge_shapes(case):
    B, Hq, Hkv, Sq, Sk, d, causal = case
    _full_case(B, Hq, Hkv, Sq, Sk, d, causal, seed=100 + Sq + Sk + d)


@pytest.mark.parametrize("causal", [False, True])
def test_key_padding_with_empty_sequences(causal):
    k_lens = torch.tensor([0, 1, 77, 256], dtype=torch.int32)
    _full_case(4, 2, 1, 256, 256, 128, causal, seed=5, k_lens=k_lens)


def test_sk_zero_all_rows_empty():
    q, k, v = W.prefill_inputs(1, 2, 2, 70, 1, 64, seed=3)
    k0 = torch.empty((1, 2, 0, 64), dtype=torch.bfloat16)
    o, lse = _run(q, k0, k0, False, 0.125)
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


@pytest.mark.parametrize("scale", [0.0, -0.2, 2.0])
def test_unusual_scales(scale):
    _full_case(1, 2, 1, 150, 150, 64, True, seed=9, scale=scale)


def test_large_magnitude_scores_stay_finite():
    # Inputs 3x unit scale: logits with std ~9 exercise the lazy rescale (the
    # exponent base moves by more than 8).  Outside the unit-scale regime the
    # absolute 1e-2 bar does not apply; the bound here follows from the
    # arithmetic: rounding O to bf16 costs up to 2^-8 |O|, and rounding P to
    # bf16 (weights normalised by the rounded sum) up to 2^-8 max|V|.
    q, k, v = W.prefill_inputs(1, 2, 2, 256, 512, 128, seed=13, value_scale=3.0)
    o, lse = _run(q, k, v, False, 1 / math.sqrt(128))
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, False, 1 / math.sqrt(128))
    og = o.double().numpy()
    assert np.isfinite(og).all() and np.isfinite(lse.numpy()).all()
    vmax = float(v.abs().max())
    bound = 2.0 ** -8 * np.abs(o_ref) + 2.0 ** -8 * vmax + 1e-3
    assert np.all(np.abs(og - o_ref) <= bound)
    rel_rms = np.linalg.norm(og - o_ref) / np.linalg.norm(o_ref)
    assert rel_rms <= 5e-3
    assert np.abs(lse.numpy() - lse_ref).max() <= 1e-3


@pytest.mark.parametrize("d,causal", [(128, False), (128, True), (64, True)])
def test_scores_rising_across_key_tiles(d, causal):
    # Key tiles scaled 1, 2.5, 5, 12: from tile to tile a row's max grows by
    # less than 8, by 8..16 and by more than 16 (log2 units), so the exponent
    # base stays put, moves one step late, and (for the last tile) the tile is
    # recomputed against its own max.  Error bound as in the test above.
    q, k, v = W.prefill_inputs(1, 2, 1, 512, 512, d, seed=29)
    f = torch.tensor([1.0, 2.5, 5.0, 12.0]).repeat_interleave(128).view(1, 1, 512, 1)
    k = (k.float() * f).to(torch.bfloat16)
    scale = 1 / math.sqrt(d)
    o, lse = _run(q, k, v, causal, scale)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, causal, scale)
    og = o.double().numpy()
    assert np.isfinite(og).all() and np.isfinite(lse.numpy()).all()
    bound = 2.0 ** -8 * np.abs(o_ref) + 2.0 ** -8 * float(v.abs().max()) + 1e-3
    assert np.all(np.abs(og - o_ref) <= bound)
    assert np.linalg.norm(og - o_ref) / np.linalg.norm(o_ref) <= 5e-3
    assert np.abs(lse.numpy() - lse_ref).max() <= 1e-3


def test_worked_example_embedded():
    # "Attention Kernel", section "Blockwise reference": scores [1, -inf, 3, -2, 0]
    # against values arange(15) as 5 x 3.  Embedded with d = 64, q = e0,
    # k_j = s_j e0 (scale 1); the -inf key becomes a padded key (k_len = 4) and
    # the finite keys are reordered [1, 3, -2, 0] (key order is irrelevant
    # without a causal mask).
    d = 64
    q = torch.zeros(1, 1, 1, d, dtype=torch.bfloat16)
    q[0, 0, 0, 0] = 1.0
    s = [1.0, 3.0, -2.0, 0.0, 5.0]
    vals = [[0, 1, 2], [6, 7, 8], [9, 10, 11], [12, 13, 14], [3, 4, 5]]
    k = torch.zeros(1, 1, 5, d, dtype=torch.bfloat16)
    v = torch.zeros(1, 1, 5, d, dtype=torch.bfloat16)
    for j in range(5):
        k[0, 0, j, 0] = s[j]
        v[0, 0, j, :3] = torch.tensor(vals[j], dtype=torch.bfloat16)
    o, lse = _run(q, k, v, False, 1.0, torch.tensor([4], dtype=torch.int32))
    expect = [5.586297614919345, 6.586297614919345, 7.586297614919346]
    np.testing.assert_allclose(o[0, 0, 0, :3].double().numpy(), expect, atol=1e-2, rtol=0)
    assert torch.all(o[0, 0, 0, 3:] == 0)
    assert abs(float(lse[0, 0, 0]) - 3.1755153626167143) < 1e-3
    o0, lse0 = _run(q, k, v, False, 1.0, torch.tensor([0], dtype=torch.int32))
    assert torch.all(o0 == 0) and torch.isneginf(lse0).all()


def test_deterministic_bitwise():
    q, k, v = W.prefill_inputs(2, 4, 2, 700, 700, 128, seed=17)
    o1, l1 = _run(q, k, v, True, 0.088)
    o2, l2 = _run(q, k, v, True, 0.088)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_gqa_equals_repeated_kv():
    q, k, v = W.prefill_inputs(1, 8, 2, 300, 300, 128, seed=19)
    o1, l1 = _run(q, k, v, True, 0.088)
    o2, l2 = _run(q, k.repeat_interleave(4, 1).contiguous(), v.repeat_interleave(4, 1).contiguous(),
                  True, 0.088)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_lse_optional_and_no_lse_output_identical():
    q, k, v = W.prefill_inputs(1, 2, 2, 256, 256, 64, seed=23)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o1, _ = attn_fwd(qd, kd, vd, True, 0.125)
    o2, l2 = attn_fwd(qd, kd, vd, True, 0.125, return_lse=False)
    torch.cuda.synchronize()
    assert l2 is None and torch.equal(o1, o2)


def test_bad_k_len_is_clamped_and_flagged():
    q, k, v = W.prefill_inputs(1, 1, 1, 128, 128, 64, seed=29)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    attn_get_device_error()  # clear
    o, lse = attn_fwd_masked(qd, kd, vd, False, 0.125,
                             k_lens=torch.tensor([1000], dtype=torch.int32, device=DEV))
    st, flags = attn_get_device_error()
    assert st != 0 and (flags & 0x4)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, False, 0.125)
    check(o.cpu(), o_ref, lse.cpu(), lse_ref, what="clamped k_len")
    st, flags = attn_get_device_error()
    assert st == 0 and flags == 0
