"""Pins for the FP8-cache decode oracle (``oracle/kv_fp8.py``), each against
something other than itself:

* E4M3 decoding against torch's float8_e4m3fn for all 256 codes (a library
  routine), plus values fixed by the format's definition;
* with per-(page, head) scales that are powers of two, every dequantised
  value is exact in bf16, so the FP8 oracle must equal the C bf16 decode
  oracle (an independent implementation) run on that bf16 cache;
* scale laws: the V scale scales O and leaves the LSE alone; a uniform K
  scale c is the softmax scale multiplied by c.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle.kv_fp8 import decode_paged_fp8, dequantize, e4m3_to_float
from exact_softmax_attention_fwd_b200 import workloads as W


def test_e4m3_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = e4m3_to_float(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2  # 0x7F and 0xFF
    np.testing.assert_array_equal(ours[~nan], ref[~nan])


def test_e4m3_values_from_the_format():
    v = e4m3_to_float(np.array([0x00, 0x80, 0x01, 0x07, 0x08, 0x38, 0xB8, 0x7E, 0xFE, 0x3C],
                               dtype=np.uint8))
    want = [0.0, -0.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 1.0, -1.0, 448.0, -448.0, 1.5]
    np.testing.assert_array_equal(v, want)


def _random_codes(shape, gen):
    c = torch.randint(0, 256, shape, generator=gen, dtype=torch.int64).to(torch.uint8)
    c[(c & 0x7F) == 0x7F] = 0x3C  # no NaN codes
    return c


@pytest.mark.parametrize("page_size,d,Hq,Hkv", [(16, 64, 4, 2), (32, 128, 8, 2), (16, 128, 2, 2)])
def test_fp8_decode_equals_bf16_oracle_on_exact_values(page_size, d, Hq, Hkv):
    gen = torch.Generator().manual_seed(31)
    lens = torch.tensor([1, 37, 0, 100], dtype=torch.int32)
    base = W.paged_inputs(lens, Hq, Hkv, d, page_size, seed=31, extra_pages=2)
    P = base.num_pages
    k8 = _random_codes((P, page_size, Hkv, d), gen)
    v8 = _random_codes((P, page_size, Hkv, d), gen)
    # powers of two keep k_scale * e4m3 exact in bf16 (3 mantissa bits)
    ks = torch.pow(2.0, torch.randint(-4, 3, (P, Hkv), generator=gen).double()).float()
    vs = torch.pow(2.0, torch.randint(-4, 3, (P, Hkv), generator=gen).double()).float()
    # the bf16 reference cache, dequantised independently of the oracle (torch's
    # float8 decode, scales broadcast per page and head)
    kd = (k8.view(torch.float8_e4m3fn).double() * ks.double()[:, None, :, None]).to(torch.bfloat16)
    vd = (v8.view(torch.float8_e4m3fn).double() * vs.double()[:, None, :, None]).to(torch.bfloat16)
    np.testing.assert_array_equal(kd.double().numpy(), dequantize(k8.numpy(), ks.numpy()))
    scale = 0.03
    o, lse = decode_paged_fp8(base.q, k8, v8, ks, vs, base.block_table, lens, scale)
    o_ref, lse_ref = oracle.decode_paged(base.q, kd, vd, base.block_table, lens, scale)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-10)
    fin = np.isfinite(lse_ref)
    np.testing.assert_allclose(lse[fin], lse_ref[fin], rtol=0, atol=1e-10)
    assert np.array_equal(np.isneginf(lse), np.isneginf(lse_ref))


def test_fp8_scale_laws():
    c = W.fp8_paged_inputs(torch.tensor([70, 5], dtype=torch.int32), 4, 2, 64, 16, seed=32)
    o, lse = decode_paged_fp8(c.q, c.k_cache, c.v_cache, c.k_scale, c.v_scale, c.block_table,
                              c.seq_lens, 0.1)
    # a power-of-two factor keeps the float32 scales exact
    o2, lse2 = decode_paged_fp8(c.q, c.k_cache, c.v_cache, c.k_scale, c.v_scale * 4.0,
                                c.block_table, c.seq_lens, 0.1)
    np.testing.assert_allclose(o2, 4.0 * o, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(lse2, lse)
    o3, lse3 = decode_paged_fp8(c.q, c.k_cache, c.v_cache, c.k_scale * 2.0, c.v_scale,
                                c.block_table, c.seq_lens, 0.05)
    np.testing.assert_allclose(o3, o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse3, lse, rtol=1e-12, atol=1e-12)


def test_fp8_generator_roundtrip_error_is_within_e4m3_rounding():
    base = W.paged_inputs(torch.tensor([64], dtype=torch.int32), 2, 2, 64, 16, seed=33)
    codes, sc = W.quantize_e4m3_per_page(base.k_cache)
    back = dequantize(codes.numpy(), sc.numpy())
    x = base.k_cache.double().numpy()
    # E4M3 keeps 3 mantissa bits: relative error <= 2^-4 on normals; absolute
    # error <= half the subnormal step (2^-10 * scale) below the normal range
    err = np.abs(back - x)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * sc.numpy()[:, None, :, None])
    assert (err <= bound * (1 + 1e-12)).all()
    assert np.abs(back).max() <= 448.0 * float(sc.double().max()) * (1 + 1e-12)


# --------------------------------------------------------------------------- block-scaled prefill

from oracle.kv_fp8 import attn_fwd_fp8, dequantize_blocks  # noqa: E402


def _codes(shape, gen):
    return _random_codes(shape, gen)


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,d,causal,k_lens", [
    (1, 2, 1, 200, 300, 64, True, None),
    (2, 4, 2, 130, 130, 64, False, [130, 90]),
    (1, 2, 2, 300, 150, 128, True, [150]),        # Sq > Sk: leading rows see no key
])
def test_fp8_prefill_equals_bf16_oracle_on_exact_values(B, Hq, Hkv, Sq, Sk, d, causal, k_lens):
    gen = torch.Generator().manual_seed(51)
    q8 = _codes((B, Hq, Sq, d), gen)
    k8 = _codes((B, Hkv, Sk, d), gen)
    v8 = _codes((B, Hkv, Sk, d), gen)

    def p2(shape):  # power-of-two block scales: dequantised values exact in bf16
        return torch.pow(2.0, torch.randint(-6, 1, shape, generator=gen).double()).float()

    qs, ks, vs = p2((B, Hq, -(-Sq // 128))), p2((B, Hkv, -(-Sk // 128))), p2((B, Hkv, -(-Sk // 128)))
    def deq(codes, sc):  # independent of the oracle: torch's float8 decode, rows of 128
        rows = sc.double().repeat_interleave(128, dim=2)[:, :, :codes.shape[2], None]
        return (codes.view(torch.float8_e4m3fn).double() * rows).to(torch.bfloat16)

    Q, K, V = deq(q8, qs), deq(k8, ks), deq(v8, vs)
    np.testing.assert_array_equal(Q.double().numpy(), dequantize_blocks(q8.numpy(), qs.numpy()))
    scale = 0.02
    o, lse = attn_fwd_fp8(q8, k8, v8, qs, ks, vs, causal, scale, k_lens=k_lens)
    o_ref, lse_ref = oracle.attn_fwd(Q, K, V, causal, scale, k_lens=k_lens)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-10)
    assert np.array_equal(np.isneginf(lse), np.isneginf(lse_ref))
    fin = np.isfinite(lse_ref)
    np.testing.assert_allclose(lse[fin], lse_ref[fin], rtol=0, atol=1e-10)


def test_fp8_prefill_scale_laws_and_block_locality():
    gen = torch.Generator().manual_seed(52)
    B, H, S, d = 1, 2, 260, 64
    q8, k8, v8 = _codes((B, H, S, d), gen), _codes((B, H, S, d), gen), _codes((B, H, S, d), gen)
    nb = -(-S // 128)
    one = torch.ones((B, H, nb))
    o, lse = attn_fwd_fp8(q8, k8, v8, one * 0.01, one * 0.01, one, True, 0.5)
    # V scale x 4 scales O; a uniform K scale x 2 is the softmax scale x 2
    o2, lse2 = attn_fwd_fp8(q8, k8, v8, one * 0.01, one * 0.01, one * 4.0, True, 0.5)
    np.testing.assert_allclose(o2, 4.0 * o, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(lse2, lse)
    o3, lse3 = attn_fwd_fp8(q8, k8, v8, one * 0.01, one * 0.02, one, True, 0.25)
    np.testing.assert_allclose(o3, o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse3, lse, rtol=1e-12, atol=1e-12)
    # a Q scale change in one block of head 0 moves only that block's rows
    for blk, lo, hi in ((0, 0, 128), (2, 256, S)):
        qs = (one * 0.01).clone()
        qs[0, 0, blk] *= 2.0
        o4, _ = attn_fwd_fp8(q8, k8, v8, qs, one * 0.01, one, True, 0.5)
        changed = np.abs(o4 - o).max(axis=-1) > 0
        assert changed[0, 0, max(lo, 1):hi].all()  # causal row 0 sees only key 0: O = v0
        assert not changed[0, 0, :lo].any() and not changed[0, 0, hi:].any()
        assert not changed[0, 1].any()


# --------------------------------------------------------------------------- paged prefill over an E4M3 cache

from oracle.kv_fp8 import attn_fwd_paged_fp8  # noqa: E402


def test_fp8_paged_prefill_equals_bf16_paged_oracle_on_exact_values():
    gen = torch.Generator().manual_seed(61)
    lq, lk = [5, 0, 40, 1], [37, 3, 100, 16]
    Hq, Hkv, d, ps = 4, 2, 64, 16
    q, cu_q, c = W.paged_prefill_inputs(lq, lk, Hq, Hkv, d, ps, seed=61)
    P = c.k_cache.shape[0]
    k8 = _random_codes((P, ps, Hkv, d), gen)
    v8 = _random_codes((P, ps, Hkv, d), gen)
    ks = torch.pow(2.0, torch.randint(-4, 3, (P, Hkv), generator=gen).double()).float()
    vs = torch.pow(2.0, torch.randint(-4, 3, (P, Hkv), generator=gen).double()).float()
    kd = (k8.view(torch.float8_e4m3fn).double() * ks.double()[:, None, :, None]).to(torch.bfloat16)
    vd = (v8.view(torch.float8_e4m3fn).double() * vs.double()[:, None, :, None]).to(torch.bfloat16)
    lens = torch.tensor(lk, dtype=torch.int32)
    for causal in (True, False):
        o, lse = attn_fwd_paged_fp8(q, k8, v8, ks, vs, c.block_table, cu_q, lens, causal, 0.05)
        o_ref, lse_ref = oracle.attn_fwd_paged(q, kd, vd, c.block_table, cu_q, lens, causal, 0.05)
        np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-10)
        fin = np.isfinite(lse_ref)
        np.testing.assert_allclose(lse[fin], lse_ref[fin], rtol=0, atol=1e-10)


def test_fp8_paged_prefill_one_query_per_sequence_is_decode():
    c = W.fp8_paged_inputs(torch.tensor([70, 1, 33], dtype=torch.int32), 8, 2, 64, 16, seed=62)
    q = c.q  # [B, Hq, d]: one new token per sequence
    cu_q = torch.arange(q.shape[0] + 1, dtype=torch.int32)
    o, lse = attn_fwd_paged_fp8(q, c.k_cache, c.v_cache, c.k_scale, c.v_scale, c.block_table,
                                cu_q, c.seq_lens, True, 0.1)
    o_d, lse_d = decode_paged_fp8(q, c.k_cache, c.v_cache, c.k_scale, c.v_scale, c.block_table,
                                  c.seq_lens, 0.1)
    np.testing.assert_allclose(o, o_d, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.T, lse_d, rtol=0, atol=1e-12)
