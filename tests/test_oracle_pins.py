"""Pins for the CPU oracle: each checks it against something other than itself.

* The worked example of "Attention Kernel", section "Blockwise reference":
  the page states the blockwise result must equal softmax(score) @ value
  (evaluated here with torch.softmax, a library routine), that an all -inf row
  returns zeros, and that mismatched score/value rows are rejected.
* Invariance of the (m, l, o) recurrence to block size and order ("Online
  softmax": any block order gives the exact merge).
* torch's scaled_dot_product_attention in float64 on tiny shapes (a library
  routine), plus a long-double evaluation written differently
  (exp(s - logsumexp)).
* Closed forms: constant V, uniform weights, causal row 0, scale 0.
* GQA == MHA with K/V repeated; key permutation invariance; paged == gathered
  contiguous ("Attention Kernel", section "验证": a contiguous cache and a
  random block table must agree).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from exact_softmax_attention_fwd_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")
NEG_INF = float("-inf")


def _golden():
    with open(GOLDEN) as f:
        g = json.load(f)
    score = [NEG_INF if s == "-inf" else float(s) for s in g["score"]]
    value = np.array(g["value"], dtype=np.float64).reshape(g["value_shape"])
    return g, score, value


# --------------------------------------------------------------------------- worked example


def test_worked_example_matches_torch_softmax():
    g, score, value = _golden()
    expected = (torch.softmax(torch.tensor(score, dtype=torch.float64), dim=0)
                @ torch.tensor(value)).numpy()
    o, lse = oracle.softmax_attend(score, value)
    np.testing.assert_allclose(o, expected, rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["expected_o"], expected, rtol=0, atol=1e-12)
    lse_ref = torch.logsumexp(torch.tensor(score, dtype=torch.float64), dim=0).item()
    assert abs(lse - lse_ref) < 1e-12
    assert abs(g["expected_lse"] - lse_ref) < 1e-12


def test_worked_example_blockwise_block2():
    g, score, value = _golden()
    o, lse = oracle.online_attend(score, value, g["block_size"])
    np.testing.assert_allclose(o, g["expected_o"], rtol=0, atol=1e-12)
    assert abs(lse - g["expected_lse"]) < 1e-12


def test_all_masked_row_is_zero_not_nan():
    _, _, value = _golden()
    row = [NEG_INF] * 5
    for o, lse in (oracle.softmax_attend(row, value), oracle.online_attend(row, value, 2)):
        assert np.array_equal(o, np.zeros(3))
        assert lse == NEG_INF


def test_mismatched_rows_rejected():
    _, score, _ = _golden()
    for fn in (lambda: oracle.softmax_attend(score, np.zeros((6, 3))),
               lambda: oracle.online_attend(score, np.zeros((6, 3)), 2)):
        with pytest.raises(oracle.OracleError) as e:
            fn()
        assert e.value.status == oracle.ERR_ARG
    with pytest.raises(oracle.OracleError):
        oracle.online_attend(score, np.zeros((5, 3)), 0)


# --------------------------------------------------------------------------- recurrence invariance


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_online_invariant_to_block_size_and_order(seed):
    rng = np.random.default_rng(seed)
    n, dv = 53, 7
    s = rng.normal(0, 3, n)
    s[rng.random(n) < 0.2] = NEG_INF
    s[10:20] = NEG_INF  # a whole block with nothing finite for several sizes
    v = rng.normal(0, 1, (n, dv))
    o_ref, lse_ref = oracle.softmax_attend(s, v)
    for bs in (1, 2, 3, 7, 16, 64, n):
        nb = -(-n // bs)
        orders = [None, list(range(nb))[::-1], list(rng.permutation(nb))]
        for order in orders:
            o, lse = oracle.online_attend(s, v, bs, order)
            np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
            assert abs(lse - lse_ref) < 1e-12


def test_online_rejects_bad_order():
    with pytest.raises(oracle.OracleError):
        oracle.online_attend([0.0, 1.0, 2.0], np.zeros((3, 2)), 1, [0, 0, 1])


# --------------------------------------------------------------------------- prefill pins


def _visible_mask(Sq, Sk, causal, klen):
    i = torch.arange(Sq)[:, None]
    j = torch.arange(Sk)[None, :]
    vis = (j < klen).expand(Sq, Sk)
    if causal:
        vis = vis & (j <= i + (klen - Sq))
    return vis


def _sdpa_reference(q, k, v, causal, scale, k_lens):
    """torch SDPA (float64, CPU) with an explicit boolean mask; empty rows -> 0/-inf."""
    B, Hq, Sq, d = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    g = Hq // Hkv
    qd, kd, vd = q.double(), k.double().repeat_interleave(g, 1), v.double().repeat_interleave(g, 1)
    o = torch.zeros(B, Hq, Sq, d, dtype=torch.float64)
    lse = torch.full((B, Hq, Sq), NEG_INF, dtype=torch.float64)
    for b in range(B):
        kl = Sk if k_lens is None else int(k_lens[b])
        vis = _visible_mask(Sq, Sk, causal, kl)
        nonempty = vis.any(-1)
        if Sk > 0 and nonempty.any():
            ob = torch.nn.functional.scaled_dot_product_attention(
                qd[b], kd[b], vd[b], attn_mask=vis, scale=scale)
            o[b][:, nonempty] = ob[:, nonempty]
            s = (qd[b] @ kd[b].transpose(-1, -2)) * scale
            s = s.masked_fill(~vis, NEG_INF)
            lse[b][:, nonempty] = torch.logsumexp(s, -1)[:, nonempty]
    return o.numpy(), lse.numpy()


def _longdouble_reference(q, k, v, causal, scale, k_lens):
    """A differently written evaluation: weights exp(s - logsumexp(s)) in long double."""
    B, Hq, Sq, d = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    g = Hq // Hkv
    qn = q.double().numpy().astype(np.longdouble)
    kn = k.double().numpy().astype(np.longdouble)
    vn = v.double().numpy().astype(np.longdouble)
    o = np.zeros((B, Hq, Sq, d), np.longdouble)
    for b in range(B):
        kl = Sk if k_lens is None else int(k_lens[b])
        vis = _visible_mask(Sq, Sk, causal, kl).numpy()
        for h in range(Hq):
            for i in range(Sq):
                js = np.nonzero(vis[i])[0]
                if js.size == 0:
                    continue
                s = np.array([np.sum(qn[b, h, i] * kn[b, h // g, j]) * scale for j in js],
                             dtype=np.longdouble)
                mx = s.max()
                lse = mx + np.log(np.sum(np.exp(s - mx)))
                w = np.exp(s - lse)
                o[b, h, i] = (w[:, None] * vn[b, h // g, js]).sum(0)
    return o.astype(np.float64)


TINY_CASES = [
    # B, Hq, Hkv, Sq, Sk, d, causal, padded
    (1, 1, 1, 1, 1, 1, False, False),
    (1, 2, 1, 5, 7, 3, False, False),
    (2, 4, 2, 6, 6, 4, True, False),
    (2, 4, 1, 7, 7, 2, True, True),
    (1, 3, 3, 4, 9, 4, True, False),   # Sq < Sk, bottom-right causal
    (2, 2, 2, 8, 5, 3, True, True),    # Sq > Sk: leading rows fully masked
    (1, 2, 2, 3, 0, 4, False, False),  # Sk = 0: every row empty
]


@pytest.mark.parametrize("case", TINY_CASES)
def test_prefill_matches_torch_sdpa_tiny(case):
    B, Hq, Hkv, Sq, Sk, d, causal, padded = case
    q, k, v = workloads.prefill_inputs(B, Hq, Hkv, Sq, Sk, d, seed=7 + Sq + Sk)
    k_lens = None
    if padded:
        k_lens = torch.tensor([max(0, Sk - 1 - b) for b in range(B)], dtype=torch.int32)
    scale = 0.37
    o, lse = oracle.attn_fwd(q, k, v, causal, scale, k_lens=k_lens)
    o_ref, lse_ref = _sdpa_reference(q, k, v, causal, scale, k_lens)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse), fin)
    np.testing.assert_allclose(lse[fin], lse_ref[fin], rtol=0, atol=1e-12)
    assert np.all(o[~fin] == 0.0)
    o_ld = _longdouble_reference(q, k, v, causal, scale, k_lens)
    np.testing.assert_allclose(o, o_ld, rtol=0, atol=1e-12)


def test_prefill_square_causal_matches_sdpa_is_causal():
    q, k, v = workloads.prefill_inputs(2, 2, 2, 9, 9, 4, seed=11)
    o, _ = oracle.attn_fwd(q, k, v, True, 0.5)
    ref = torch.nn.functional.scaled_dot_product_attention(q.double(), k.double(), v.double(),
                                                           is_causal=True, scale=0.5)
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)


def test_prefill_constant_values():
    q, k, _ = workloads.prefill_inputs(1, 2, 2, 6, 6, 8, seed=3)
    v = torch.full((1, 2, 6, 8), 1.75, dtype=torch.bfloat16)
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, causal, 0.3)
        np.testing.assert_allclose(o, 1.75, rtol=0, atol=1e-12)
        assert np.all(np.isfinite(lse))


def test_prefill_uniform_weights_closed_form():
    # q = 0 makes every visible score 0: O is the mean of the visible V rows and
    # LSE = ln(number of visible keys).
    _, k, v = workloads.prefill_inputs(1, 1, 1, 5, 5, 4, seed=5)
    q = torch.zeros(1, 1, 5, 4, dtype=torch.bfloat16)
    o, lse = oracle.attn_fwd(q, k, v, True, 1.0)
    vd = v.double().numpy()[0, 0]
    for i in range(5):
        np.testing.assert_allclose(o[0, 0, i], vd[: i + 1].mean(0), rtol=0, atol=1e-12)
        assert abs(lse[0, 0, i] - math.log(i + 1)) < 1e-12
    # scale = 0 does the same for any q
    q2, _, _ = workloads.prefill_inputs(1, 1, 1, 5, 5, 4, seed=6)
    o2, lse2 = oracle.attn_fwd(q2, k, v, False, 0.0)
    np.testing.assert_allclose(o2[0, 0], np.broadcast_to(vd.mean(0), (5, 4)), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2, math.log(5), rtol=0, atol=1e-12)


def test_prefill_causal_row0_sees_only_key0():
    q, k, v = workloads.prefill_inputs(1, 2, 2, 4, 4, 8, seed=9)
    o, lse = oracle.attn_fwd(q, k, v, True, 0.25)
    for h in range(2):
        np.testing.assert_allclose(o[0, h, 0], v.double().numpy()[0, h, 0], rtol=0, atol=1e-12)
        s00 = 0.25 * float((q.double()[0, h, 0] * k.double()[0, h, 0]).sum())
        assert abs(lse[0, h, 0] - s00) < 1e-12


def test_prefill_gqa_equals_repeated_mha():
    q, k, v = workloads.prefill_inputs(2, 8, 2, 6, 10, 4, seed=21)
    o, lse = oracle.attn_fwd(q, k, v, True, 0.5)
    o2, lse2 = oracle.attn_fwd(q, k.repeat_interleave(4, 1), v.repeat_interleave(4, 1), True, 0.5)
    np.testing.assert_allclose(o, o2, rtol=0, atol=0)
    np.testing.assert_allclose(lse, lse2, rtol=0, atol=0)


def test_prefill_noncausal_key_permutation_invariance():
    q, k, v = workloads.prefill_inputs(1, 2, 1, 4, 12, 4, seed=31)
    perm = torch.randperm(12, generator=torch.Generator().manual_seed(0))
    o, lse = oracle.attn_fwd(q, k, v, False, 0.5)
    o2, lse2 = oracle.attn_fwd(q, k[:, :, perm].contiguous(), v[:, :, perm].contiguous(), False, 0.5)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-12)


def test_prefill_padding_equals_truncation_noncausal():
    q, k, v = workloads.prefill_inputs(2, 2, 2, 5, 11, 4, seed=41)
    k_lens = torch.tensor([7, 11], dtype=torch.int32)
    o, lse = oracle.attn_fwd(q, k, v, False, 0.5, k_lens=k_lens)
    for b, kl in enumerate(k_lens.tolist()):
        ob, lb = oracle.attn_fwd(q[b:b + 1], k[b:b + 1, :, :kl].contiguous(),
                                 v[b:b + 1, :, :kl].contiguous(), False, 0.5)
        np.testing.assert_allclose(o[b], ob[0], rtol=0, atol=0)
        np.testing.assert_allclose(lse[b], lb[0], rtol=0, atol=0)


def test_prefill_bottom_right_padding_masks_leading_rows():
    q, k, v = workloads.prefill_inputs(1, 1, 1, 8, 8, 4, seed=43)
    o, lse = oracle.attn_fwd(q, k, v, True, 0.5, k_lens=torch.tensor([5], dtype=torch.int32))
    # rows i < Sq - k_len = 3 have no visible key
    assert np.all(o[0, 0, :3] == 0) and np.all(lse[0, 0, :3] == NEG_INF)
    assert np.all(np.isfinite(lse[0, 0, 3:]))
    # the last row sees exactly keys 0..4
    ob, _ = oracle.attn_fwd(q[:, :, 7:8].contiguous(), k[:, :, :5].contiguous(),
                            v[:, :, :5].contiguous(), False, 0.5)
    np.testing.assert_allclose(o[0, 0, 7], ob[0, 0, 0], rtol=0, atol=0)


def test_prefill_row_subset_matches_full():
    q, k, v = workloads.prefill_inputs(2, 4, 2, 7, 9, 4, seed=51)
    o, lse = oracle.attn_fwd(q, k, v, True, 0.5)
    rows = workloads.sample_rows(2, 4, 7, 13, seed=1)
    o_s, lse_s = oracle.attn_fwd(q, k, v, True, 0.5, rows=rows, n_threads=3)
    np.testing.assert_array_equal(o_s, o.reshape(-1, 4)[rows.numpy()])
    np.testing.assert_array_equal(lse_s, lse.reshape(-1)[rows.numpy()])


def test_prefill_rejects_bad_args():
    q, k, v = workloads.prefill_inputs(1, 3, 2, 2, 2, 4, seed=1)
    with pytest.raises(oracle.OracleError):
        oracle.attn_fwd(q, k, v, False, 1.0)  # Hq % Hkv != 0


# --------------------------------------------------------------------------- paged decode pins


def _gather_contiguous(inp, b, Hkv, d):
    n = int(inp.seq_lens[b])
    ks, vs = [], []
    for t in range(n):
        page = int(inp.block_table[b, t // inp.page_size])
        ks.append(inp.k_cache[page, t % inp.page_size])
        vs.append(inp.v_cache[page, t % inp.page_size])
    if n == 0:
        return (torch.zeros(1, Hkv, 0, d, dtype=torch.bfloat16),) * 2
    return (torch.stack(ks, 1).unsqueeze(0).contiguous(),   # [1, Hkv, n, d]
            torch.stack(vs, 1).unsqueeze(0).contiguous())


def test_decode_paged_matches_prefill_on_gathered_kv():
    lens = torch.tensor([1, 16, 17, 40, 0, 33], dtype=torch.int32)
    Hq, Hkv, d = 8, 2, 4
    inp = workloads.paged_inputs(lens, Hq, Hkv, d, page_size=16, seed=61, extra_pages=3)
    o, lse = oracle.decode_paged(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.seq_lens, 0.5)
    for b in range(len(lens)):
        kb, vb = _gather_contiguous(inp, b, Hkv, d)
        if int(lens[b]) == 0:
            assert np.all(o[b] == 0) and np.all(lse[b] == NEG_INF)
            continue
        ob, lb = oracle.attn_fwd(inp.q[b].reshape(1, Hq, 1, d).contiguous(), kb, vb, False, 0.5)
        np.testing.assert_allclose(o[b], ob[0, :, 0], rtol=0, atol=0)
        np.testing.assert_allclose(lse[b], lb[0, :, 0], rtol=0, atol=0)
        # and against the library routine
        ref = torch.nn.functional.scaled_dot_product_attention(
            inp.q[b].double().reshape(1, Hq, 1, d),
            kb.double().repeat_interleave(Hq // Hkv, 1), vb.double().repeat_interleave(Hq // Hkv, 1),
            scale=0.5)
        np.testing.assert_allclose(o[b], ref[0, :, 0].numpy(), rtol=0, atol=1e-12)


def test_decode_contiguous_vs_permuted_pages():
    lens = torch.tensor([5, 31, 64], dtype=torch.int32)
    a = workloads.paged_inputs(lens, 4, 2, 8, 16, seed=71, contiguous=True)
    b = workloads.paged_inputs(lens, 4, 2, 8, 16, seed=71, contiguous=False)
    # same logical cache content: move b's pages into a's physical order
    kc = torch.empty_like(a.k_cache)
    vc = torch.empty_like(a.v_cache)
    for s in range(3):
        for p in range(-(-int(lens[s]) // 16)):
            kc[int(b.block_table[s, p])] = a.k_cache[int(a.block_table[s, p])]
            vc[int(b.block_table[s, p])] = a.v_cache[int(a.block_table[s, p])]
    oa, la = oracle.decode_paged(a.q, a.k_cache, a.v_cache, a.block_table, lens, 0.3)
    ob, lb = oracle.decode_paged(a.q, kc, vc, b.block_table, lens, 0.3)
    np.testing.assert_array_equal(oa, ob)
    np.testing.assert_array_equal(la, lb)


def test_decode_single_token_returns_v0():
    inp = workloads.paged_inputs(torch.tensor([1], dtype=torch.int32), 4, 2, 8, 16, seed=81)
    o, lse = oracle.decode_paged(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.seq_lens, 0.5)
    page = int(inp.block_table[0, 0])
    for h in range(4):
        np.testing.assert_allclose(o[0, h], inp.v_cache[page, 0, h // 2].double().numpy(),
                                   rtol=0, atol=0)


def test_decode_bad_page_id_reported():
    inp = workloads.paged_inputs(torch.tensor([20], dtype=torch.int32), 2, 1, 4, 16, seed=91)
    tbl = inp.block_table.clone()
    tbl[0, 1] = inp.num_pages + 5
    with pytest.raises(oracle.OracleError) as e:
        oracle.decode_paged(inp.q, inp.k_cache, inp.v_cache, tbl, inp.seq_lens, 0.5)
    assert e.value.status == oracle.ERR_TABLE


# --------------------------------------------------------------------------- ragged batches
# "Attention Kernel", section "Paged 与 ragged KV": a ragged batch is a list of
# sequences given by cumulative lengths; nothing crosses a sequence boundary.


def _packed(x):
    """[B, H, S, d] -> packed token-major [B*S, H, d]."""
    B, H, S, d = x.shape
    return x.permute(0, 2, 1, 3).reshape(B * S, H, d).contiguous()


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equal_lengths_equals_batched(causal):
    B, Hq, Hkv, S, d = 3, 4, 2, 23, 8
    q, k, v = workloads.prefill_inputs(B, Hq, Hkv, S, S, d, seed=41)
    cu = workloads.cu_seqlens([S] * B)
    o, lse = oracle.attn_fwd_varlen(_packed(q), _packed(k), _packed(v), cu, cu, causal, 0.3)
    ob, lb = oracle.attn_fwd(q, k, v, causal, 0.3)
    np.testing.assert_array_equal(o, ob.transpose(0, 2, 1, 3).reshape(B * S, Hq, d))
    np.testing.assert_array_equal(lse, lb.transpose(1, 0, 2).reshape(Hq, B * S))


def test_varlen_sequences_do_not_see_each_other():
    # changing every token of sequence 1 leaves sequences 0 and 2 bit-identical
    lens = [7, 12, 5]
    q, k, v, cu_q, cu_k = workloads.varlen_inputs(lens, lens, 2, 1, 4, seed=43)
    o, lse = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, True, 0.5)
    k2, v2 = k.clone(), v.clone()
    k2[7:19] = -k2[7:19] * 3
    v2[7:19] = v2[7:19] + 7
    o2, lse2 = oracle.attn_fwd_varlen(q, k2, v2, cu_q, cu_k, True, 0.5)
    for a, b in ((0, 7), (19, 24)):
        np.testing.assert_array_equal(o[a:b], o2[a:b])
        np.testing.assert_array_equal(lse[:, a:b], lse2[:, a:b])
    assert not np.array_equal(o[7:19], o2[7:19])


def test_varlen_empty_query_and_key_ranges():
    # sequence 1 has no query (nothing written: NaN), sequence 2 no key (O = 0, LSE = -inf)
    lens_q, lens_k = [4, 0, 3], [4, 6, 0]
    q, k, v, cu_q, cu_k = workloads.varlen_inputs(lens_q, lens_k, 2, 2, 4, seed=47)
    o, lse = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, False, 0.5)
    assert np.isfinite(o[:4]).all() and np.isfinite(lse[:, :4]).all()
    assert np.array_equal(o[4:7], np.zeros((3, 2, 4)))
    assert np.isneginf(lse[:, 4:7]).all()


def test_varlen_worked_example_masked_key_is_the_next_sequence():
    # The worked example with its -inf key realised as a sequence boundary: the
    # row sees keys [1, 3, -2, 0] (values as in the golden file, reordered);
    # the key after them, with value [3, 4, 5], is the first key of the next
    # sequence and must not contribute.
    g, _, value = _golden()
    d = 4
    s = [1.0, 3.0, -2.0, 0.0, 5.0]
    rows = [0, 2, 3, 4, 1]  # golden value rows for those keys
    q = torch.zeros(2, 1, d, dtype=torch.bfloat16)
    q[:, 0, 0] = 1.0
    k = torch.zeros(5, 1, d, dtype=torch.bfloat16)
    v = torch.zeros(5, 1, d, dtype=torch.bfloat16)
    for j in range(5):
        k[j, 0, 0] = s[j]
        v[j, 0, :3] = torch.tensor(value[rows[j]], dtype=torch.bfloat16)
    cu_q = torch.tensor([0, 1, 2], dtype=torch.int32)
    cu_k = torch.tensor([0, 4, 5], dtype=torch.int32)
    o, lse = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, False, 1.0)
    np.testing.assert_allclose(o[0, 0, :3], g["expected_o"], rtol=0, atol=1e-12)
    assert abs(lse[0, 0] - g["expected_lse"]) < 1e-12
    np.testing.assert_allclose(o[1, 0, :3], value[1], rtol=0, atol=0)  # one key: O = its value
    assert lse[0, 1] == 5.0


def test_varlen_bottom_right_causal_last_row_sees_every_key():
    # len_q < len_k: the last query row of a causal sequence sees all of its
    # keys, so it equals the non-causal result; the first row sees
    # len_k - len_q + 1 keys.
    lens_q, lens_k = [3, 5], [9, 5]
    q, k, v, cu_q, cu_k = workloads.varlen_inputs(lens_q, lens_k, 2, 1, 4, seed=53)
    oc, lc = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, True, 0.7)
    on, ln = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, False, 0.7)
    np.testing.assert_array_equal(oc[2], on[2])
    np.testing.assert_array_equal(oc[7], on[7])
    # first row of sequence 0 == non-causal attention over its first 7 keys
    o7, l7 = oracle.attn_fwd_varlen(q[:1], k[:7], v[:7], [0, 1], [0, 7], False, 0.7)
    np.testing.assert_array_equal(oc[0], o7[0])


# --------------------------------------------------------------------------- paged prefill
# "Attention Kernel", section "Paged 与 ragged KV": key token t of a sequence is
# at offset t mod page_size of the physical page block_table[b][t // page_size].


def test_paged_prefill_contiguous_pages_equal_ragged():
    lens_q, lens_k = [5, 3, 0, 9], [21, 3, 7, 40]
    q, cu_q, c = workloads.paged_prefill_inputs(lens_q, lens_k, 4, 2, 8, 16, seed=83,
                                                contiguous=True)
    o, lse = oracle.attn_fwd_paged(q, c.k_cache, c.v_cache, c.block_table, cu_q, c.seq_lens,
                                   True, 0.4)
    # with contiguous placement the keys of sequence b are the pool's rows in order
    pool_k = c.k_cache.reshape(-1, 2, 8)
    pool_v = c.v_cache.reshape(-1, 2, 8)
    starts = [0]
    for n in lens_k:
        starts.append(starts[-1] + 16 * (-(-n // 16)))
    ks = torch.cat([pool_k[starts[b]:starts[b] + lens_k[b]] for b in range(4)])
    vs = torch.cat([pool_v[starts[b]:starts[b] + lens_k[b]] for b in range(4)])
    o2, l2 = oracle.attn_fwd_varlen(q, ks, vs, cu_q, workloads.cu_seqlens(lens_k), True, 0.4)
    np.testing.assert_array_equal(np.nan_to_num(o, nan=7.0), np.nan_to_num(o2, nan=7.0))
    np.testing.assert_array_equal(np.nan_to_num(lse, nan=7.0), np.nan_to_num(l2, nan=7.0))


def test_paged_prefill_permuted_pages_equal_contiguous():
    lens_q, lens_k = [4, 6], [50, 33]
    q, cu_q, cc = workloads.paged_prefill_inputs(lens_q, lens_k, 2, 1, 4, 16, seed=89,
                                                 contiguous=True)
    _, _, cp = workloads.paged_prefill_inputs(lens_q, lens_k, 2, 1, 4, 16, seed=89)
    # move the contiguous pool's pages to the permuted placement
    k2 = torch.empty_like(cc.k_cache)
    v2 = torch.empty_like(cc.v_cache)
    for b in range(2):
        n = -(-lens_k[b] // 16)
        for lp in range(n):
            k2[cp.block_table[b, lp]] = cc.k_cache[cc.block_table[b, lp]]
            v2[cp.block_table[b, lp]] = cc.v_cache[cc.block_table[b, lp]]
    a = oracle.attn_fwd_paged(q, cc.k_cache, cc.v_cache, cc.block_table, cu_q, cc.seq_lens, True,
                              0.5)
    b_ = oracle.attn_fwd_paged(q, k2, v2, cp.block_table, cu_q, cp.seq_lens, True, 0.5)
    np.testing.assert_array_equal(a[0], b_[0])
    np.testing.assert_array_equal(a[1], b_[1])


def test_paged_prefill_single_token_equals_decode_oracle():
    # one new token per sequence sees every key: the C decode oracle's result
    lens_k = [1, 17, 64, 100]
    q, cu_q, c = workloads.paged_prefill_inputs([1] * 4, lens_k, 4, 2, 16, 16, seed=97)
    o, lse = oracle.attn_fwd_paged(q, c.k_cache, c.v_cache, c.block_table, cu_q, c.seq_lens,
                                   True, 0.3)
    od, ld = oracle.decode_paged(q, c.k_cache, c.v_cache, c.block_table, c.seq_lens, 0.3)
    np.testing.assert_allclose(o, od, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ld.T, rtol=0, atol=1e-12)


def test_paged_prefill_bad_page_is_reported():
    q, cu_q, c = workloads.paged_prefill_inputs([2], [20], 2, 1, 4, 16, seed=101)
    tbl = c.block_table.clone()
    tbl[0, 1] = c.k_cache.shape[0]
    with pytest.raises(oracle.OracleError):
        oracle.attn_fwd_paged(q, c.k_cache, c.v_cache, tbl, cu_q, c.seq_lens, True, 0.3)


def test_varlen_token_subset_equals_full_evaluation():
    lens_q, lens_k = [9, 0, 14, 3], [12, 5, 14, 0]
    q, k, v, cu_q, cu_k = workloads.varlen_inputs(lens_q, lens_k, 3, 1, 4, seed=137)
    o, lse = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, True, 0.6)
    tok = np.array([25, 0, 8, 9, 13, 24, 22])
    os_, ls_ = oracle.attn_fwd_varlen(q, k, v, cu_q, cu_k, True, 0.6, tokens=tok)
    np.testing.assert_array_equal(os_, o[tok])
    np.testing.assert_array_equal(ls_, lse[:, tok])


# --------------------------------------------------------------------------- programmable masks
# "Attention Kernel", section "可编程 mask": causal, sliding window, document
# boundaries, prefix-LM.  Window w: the row at key position p sees keys (p-w, p];
# prefix P: keys below P are visible to every row (both with the causal mask).


def _sdpa_masked(q, k, v, scale, visible):
    """torch SDPA in float64 with an explicit boolean mask [Sq, Sk] (True = visible)."""
    g = q.shape[1] // k.shape[1]
    kk = k.double().repeat_interleave(g, dim=1)
    vv = v.double().repeat_interleave(g, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(q.double(), kk, vv, attn_mask=visible,
                                                         scale=scale)
    s = torch.einsum("bhqd,bhkd->bhqk", q.double(), kk) * scale
    lse = torch.logsumexp(s.masked_fill(~visible, float("-inf")), dim=-1)
    return o.numpy(), lse.numpy()


@pytest.mark.parametrize("Sq,Sk,window", [(9, 9, 3), (5, 12, 4), (12, 12, 1), (7, 7, 20)])
def test_sliding_window_against_sdpa(Sq, Sk, window):
    q, k, v = workloads.prefill_inputs(1, 4, 2, Sq, Sk, 8, seed=139)
    o, lse = oracle.attn_fwd(q, k, v, True, 0.4, window=window)
    i = torch.arange(Sq)[:, None] + (Sk - Sq)
    j = torch.arange(Sk)[None, :]
    vis = (j <= i) & (j > i - window)  # every row keeps at least its diagonal key
    ro, rl = _sdpa_masked(q, k, v, 0.4, vis)
    np.testing.assert_allclose(o, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)


def test_window_one_is_the_diagonal_key_and_wide_window_is_causal():
    q, k, v = workloads.prefill_inputs(1, 2, 1, 11, 11, 8, seed=149)
    o, lse = oracle.attn_fwd(q, k, v, True, 0.3, window=1)
    vv = v.double().numpy()[0, 0]
    s = (q.double() @ k.double().transpose(-1, -2)).numpy()[0] * 0.3
    for h in range(2):
        np.testing.assert_allclose(o[0, h], vv, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[0, h], np.diagonal(s[h]), rtol=0, atol=1e-12)
    oc, lc = oracle.attn_fwd(q, k, v, True, 0.3)
    ow, lw = oracle.attn_fwd(q, k, v, True, 0.3, window=11)
    np.testing.assert_array_equal(oc, ow)
    np.testing.assert_array_equal(lc, lw)


@pytest.mark.parametrize("prefix", [1, 4, 9])
def test_prefix_lm_against_sdpa(prefix):
    q, k, v = workloads.prefill_inputs(1, 2, 2, 9, 9, 8, seed=151)
    o, lse = oracle.attn_fwd(q, k, v, True, 0.5, prefix=prefix)
    i = torch.arange(9)[:, None]
    j = torch.arange(9)[None, :]
    ro, rl = _sdpa_masked(q, k, v, 0.5, (j <= i) | (j < prefix))
    np.testing.assert_allclose(o, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)
    if prefix >= 9:  # every key visible: non-causal attention
        on, ln = oracle.attn_fwd(q, k, v, False, 0.5)
        np.testing.assert_array_equal(o, on)


def test_window_and_prefix_together_are_rejected():
    q, k, v = workloads.prefill_inputs(1, 1, 1, 4, 4, 8, seed=157)
    with pytest.raises(oracle.OracleError):
        oracle.attn_fwd(q, k, v, True, 0.5, window=2, prefix=2)
    with pytest.raises(oracle.OracleError):
        oracle.attn_fwd(q, k, v, False, 0.5, window=2)


def test_document_mask_is_the_ragged_batch_of_its_documents():
    # a sequence of three documents, each attending causally within itself, is
    # the ragged batch of the documents (cumulative lengths at the boundaries)
    docs = [5, 8, 3]
    q, k, v, cu, _ = workloads.varlen_inputs(docs, docs, 2, 1, 8, seed=163)
    o, lse = oracle.attn_fwd_varlen(q, k, v, cu, cu, True, 0.4)
    doc = torch.repeat_interleave(torch.arange(3), torch.tensor(docs))
    i = torch.arange(16)[:, None]
    j = torch.arange(16)[None, :]
    vis = (doc[:, None] == doc[None, :]) & (j <= i)
    ro, rl = _sdpa_masked(q.permute(1, 0, 2)[None], k.permute(1, 0, 2)[None],
                          v.permute(1, 0, 2)[None], 0.4, vis)
    np.testing.assert_allclose(o, ro[0].transpose(1, 0, 2), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl[0], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------- block-sparse masks
# "Attention Kernel", section "可编程 mask": block-level sparsity decides which
# tiles are skipped entirely.  A zero entry of the [B, 1 or H, Sq/128, Sk/128]
# block mask hides the whole 128 x 128 block.


@pytest.mark.parametrize("causal,heads", [(False, 1), (True, 4)])
def test_block_mask_against_sdpa(causal, heads):
    B, Hq, Hkv, Sq, Sk, d = 1, 4, 2, 300, 420, 8
    q, k, v = workloads.prefill_inputs(B, Hq, Hkv, Sq, Sk, d, seed=191)
    g = torch.Generator().manual_seed(193)
    bm = (torch.rand(B, heads, 3, 4, generator=g) < 0.6).to(torch.uint8)
    bm[..., 0] = 1  # every row keeps its first key block
    o, lse = oracle.attn_fwd(q, k, v, causal, 0.3, block_mask=bm)
    blk = bm.repeat_interleave(128, 2).repeat_interleave(128, 3)[:, :, :Sq, :Sk].bool()
    vis = blk.expand(B, Hq, Sq, Sk)
    if causal:
        i = torch.arange(Sq)[:, None] + (Sk - Sq)
        vis = vis & (torch.arange(Sk)[None, :] <= i)
    ro, rl = _sdpa_masked(q, k, v, 0.3, vis)
    np.testing.assert_allclose(o, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)


def test_block_mask_all_ones_is_no_mask_and_empty_rows_are_zero():
    q, k, v = workloads.prefill_inputs(2, 2, 2, 200, 300, 8, seed=197)
    ones = np.ones((2, 1, 2, 3), np.uint8)
    a = oracle.attn_fwd(q, k, v, True, 0.5, block_mask=ones)
    b_ = oracle.attn_fwd(q, k, v, True, 0.5)
    np.testing.assert_array_equal(a[0], b_[0])
    np.testing.assert_array_equal(a[1], b_[1])
    bm = ones.copy()
    bm[1, 0, 1, :] = 0  # sequence 1, query rows 128..199: no visible block
    o, lse = oracle.attn_fwd(q, k, v, False, 0.5, block_mask=bm)
    assert np.array_equal(o[1, :, 128:], np.zeros_like(o[1, :, 128:]))
    assert np.isneginf(lse[1, :, 128:]).all()
