"""CPU oracle for decode over an FP8 (e4m3) paged KV cache -- TEST INFRASTRUCTURE ONLY.

Plain float64 numpy.  The cache holds one byte per element in the OCP 8-bit
floating-point format E4M3 (1 sign bit, 4 exponent bits with bias 7, 3
mantissa bits; exponent field 0 encodes subnormals m * 2^-9; the all-ones
exponent with all-ones mantissa is NaN; there is no infinity), plus one fp32
scale per (physical page, KV head) for K and one for V.  The dequantised
cache is
    K[page, row, h, :] = k_scale[page, h] * e4m3(k_bytes[page, row, h, :])
and likewise V; decode is then exact softmax attention of one query row per
(sequence, query head) over the sequence's tokens, gathered through the block
table exactly as for a bf16 cache.

Sources (page title, section):
  * "Attention Kernel" -- "Paged 与 ragged KV" (token t lives in block
    t / page_size at offset t mod page_size; the block table maps it to a
    physical page) and "正确性契约" (the cache quantisation schema is part of
    the kernel's contract, next to page size and valid-token counts).
  * "Attention 算子加速史" -- section 3 (FP8 operands with scale factors on
    FlashAttention-3) and section 4 (paged decode).
  * "Attention Kernel" -- "问题与成本" and "Online softmax" (the attention
    itself, and the zero output / -inf LSE of a row with no key).

``attn_fwd_fp8`` states prefill over E4M3 Q, K and V with block scaling
("Attention 算子加速史", section 3: FlashAttention-3 pairs FP8 with block-level
adaptive scaling; the pages give no block shape): one fp32 scale per (batch,
head, block of 128 consecutive rows) of each tensor, value = scale * e4m3(code),
then exact masked attention of the dequantised values (the masking rules of
the bf16 prefill: key lengths, bottom-right causal alignment, zero output and
-inf LSE for a row with no visible key).

Pinned in ``tests/test_oracle_fp8_pins.py``: the E4M3 decoding against torch's
float8_e4m3fn for all 256 codes; with power-of-two scales, whose dequantised
values are exact in bf16, against the C bf16 decode and prefill oracles on
those values; scale laws (a V scale scales O, a K scale acts as the softmax
scale); per-page scales applied to the right pages and a block scale confined
to its 128 rows.  ``attn_fwd_paged_fp8`` (queries appended to an E4M3 paged
cache) is pinned against the C paged-prefill oracle the same way and, with one
query per sequence, against ``decode_paged_fp8``.
"""
from __future__ import annotations

import numpy as np


def e4m3_to_float(codes) -> np.ndarray:
    """Values of E4M3 bytes (uint8 array) as float64: sign * 2^(e-7) * (1 + m/8)
    for exponent field e > 0, sign * m * 2^-9 for e = 0, NaN for 0x7F / 0xFF."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = sign * np.ldexp(1.0 + m / 8.0, e - 7)
    sub = sign * m * 2.0 ** -9
    out = np.where(e == 0, sub, normal)
    return np.where((c & 0x7F) == 0x7F, np.nan, out)


def dequantize(cache_bytes, scales) -> np.ndarray:
    """[num_pages, page_size, Hkv, d] bytes and [num_pages, Hkv] scales -> float64 values."""
    vals = e4m3_to_float(cache_bytes)
    s = np.asarray(scales, dtype=np.float64)
    return vals * s[:, None, :, None]


def _f64(x) -> np.ndarray:
    if isinstance(x, np.ndarray):
        if x.dtype == np.uint16:  # bf16 bit patterns
            return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        return x.astype(np.float64)
    return x.detach().cpu().double().numpy()


def decode_paged_fp8(q, k_bytes, v_bytes, k_scale, v_scale, block_table, seq_lens, scale):
    """One query row per (sequence, query head) over an FP8 paged cache.

    q [B, Hq, d] (bf16 tensor or floats); k_bytes, v_bytes uint8 [num_pages,
    page_size, Hkv, d]; k_scale, v_scale [num_pages, Hkv]; block_table int
    [B, max_pages]; seq_lens [B].  Returns (o [B, Hq, d], lse [B, Hq]) float64;
    a sequence of length 0 gives o = 0 and lse = -inf.
    """
    Q = _f64(q)
    kb = np.asarray(k_bytes.cpu().numpy() if hasattr(k_bytes, "cpu") else k_bytes, np.uint8)
    vb = np.asarray(v_bytes.cpu().numpy() if hasattr(v_bytes, "cpu") else v_bytes, np.uint8)
    ks = np.asarray(k_scale.cpu().numpy() if hasattr(k_scale, "cpu") else k_scale, np.float64)
    vs = np.asarray(v_scale.cpu().numpy() if hasattr(v_scale, "cpu") else v_scale, np.float64)
    tbl = np.asarray(block_table.cpu().numpy() if hasattr(block_table, "cpu") else block_table)
    lens = np.asarray(seq_lens.cpu().numpy() if hasattr(seq_lens, "cpu") else seq_lens)
    B, Hq, d = Q.shape
    num_pages, page_size, Hkv, dk = kb.shape
    if dk != d or vb.shape != kb.shape or ks.shape != (num_pages, Hkv) or vs.shape != ks.shape:
        raise ValueError("cache / scale shapes disagree")
    g = Hq // Hkv
    K = dequantize(kb, ks)
    V = dequantize(vb, vs)
    o = np.zeros((B, Hq, d))
    lse = np.full((B, Hq), -np.inf)
    for b in range(B):
        n = int(lens[b])
        if n == 0:
            continue
        t = np.arange(n)
        pages = tbl[b, t // page_size]
        if (pages < 0).any() or (pages >= num_pages).any():
            raise ValueError("block table entry out of range")
        rows = t % page_size
        for hq in range(Hq):
            h = hq // g
            kk = K[pages, rows, h, :]          # [n, d]
            vv = V[pages, rows, h, :]
            s = scale * (kk @ Q[b, hq])
            mx = s.max()
            w = np.exp(s - mx)
            o[b, hq] = (w @ vv) / w.sum()
            lse[b, hq] = mx + np.log(w.sum())
    return o, lse


def dequantize_blocks(codes, scales, block: int = 128) -> np.ndarray:
    """[B, H, S, d] E4M3 bytes and [B, H, ceil(S/block)] scales -> float64 values."""
    vals = e4m3_to_float(np.asarray(codes, dtype=np.uint8))
    sc = np.asarray(scales, dtype=np.float64)
    S = vals.shape[2]
    if sc.shape != vals.shape[:2] + (-(-S // block),):
        raise ValueError("scales must be [B, H, ceil(S / block)]")
    return vals * np.repeat(sc, block, axis=2)[:, :, :S, None]


def attn_fwd_fp8(q_codes, k_codes, v_codes, q_scale, k_scale, v_scale, causal, scale,
                 k_lens=None):
    """Prefill over block-scaled E4M3 inputs, float64.

    q_codes [B, Hq, Sq, d], k_codes / v_codes [B, Hkv, Sk, d] uint8; scales
    [B, H, ceil(S/128)] for each tensor.  Key j is visible to row i iff
    j < k_len and (causal => j <= i + k_len - Sq).  Returns (o [B, Hq, Sq, d],
    lse [B, Hq, Sq]).
    """
    def arr(x):
        return np.asarray(x.cpu().numpy() if hasattr(x, "cpu") else x)
    Q = dequantize_blocks(arr(q_codes), arr(q_scale))
    K = dequantize_blocks(arr(k_codes), arr(k_scale))
    V = dequantize_blocks(arr(v_codes), arr(v_scale))
    B, Hq, Sq, d = Q.shape
    _, Hkv, Sk, _ = K.shape
    if K.shape != V.shape or K.shape[0] != B or K.shape[3] != d or Hq % Hkv:
        raise ValueError("q/k/v shapes disagree")
    g = Hq // Hkv
    o = np.zeros((B, Hq, Sq, d))
    lse = np.full((B, Hq, Sq), -np.inf)
    i = np.arange(Sq)[:, None]
    j = np.arange(Sk)[None, :]
    for b in range(B):
        kl = Sk if k_lens is None else int(arr(k_lens)[b])
        vis = j < kl
        if causal:
            vis = vis & (j <= i + (kl - Sq))
        live = vis.any(axis=1)
        for hq in range(Hq):
            s = np.where(vis, scale * (Q[b, hq] @ K[b, hq // g].T), -np.inf)
            m = np.where(live, s.max(axis=1), 0.0)
            w = np.where(vis, np.exp(s - m[:, None]), 0.0)
            den = w.sum(axis=1)
            den_safe = np.where(live, den, 1.0)
            o[b, hq] = np.where(live[:, None], (w @ V[b, hq // g]) / den_safe[:, None], 0.0)
            lse[b, hq] = np.where(live, m + np.log(den_safe), -np.inf)
    return o, lse


def attn_fwd_paged_fp8(q, k_bytes, v_bytes, k_scale, v_scale, block_table, cu_seqlens_q,
                       seq_lens_k, causal, scale):
    """Packed queries appended to an E4M3 paged cache (per-(page, KV head) scales).

    q [total_q, Hq, d] (bf16 tensor or floats); caches and scales as in
    ``decode_paged_fp8``; cu_seqlens_q [B + 1]; seq_lens_k [B].  Key token t of
    sequence b is the dequantised row (block_table[b][t // page_size],
    t % page_size); the sequence's len_q queries are its last len_q positions
    (bottom-right causal rule).  Returns (o [total_q, Hq, d], lse [Hq, total_q])
    float64; a sequence with no key gives o = 0, lse = -inf.
    """
    def arr(x):
        return np.asarray(x.cpu().numpy() if hasattr(x, "cpu") else x)
    Q = _f64(q)
    K = dequantize(arr(k_bytes), arr(k_scale))
    V = dequantize(arr(v_bytes), arr(v_scale))
    tbl, cq, lens = arr(block_table), arr(cu_seqlens_q), arr(seq_lens_k)
    num_pages, page_size, Hkv, d = K.shape
    total_q, Hq, _ = Q.shape
    g = Hq // Hkv
    o = np.zeros((total_q, Hq, d))
    lse = np.full((Hq, total_q), -np.inf)
    for b in range(len(lens)):
        qa, qe, n = int(cq[b]), int(cq[b + 1]), int(lens[b])
        lq = qe - qa
        if lq == 0 or n == 0:
            continue
        t = np.arange(n)
        pages = tbl[b, t // page_size]
        if (pages < 0).any() or (pages >= num_pages).any():
            raise ValueError("block table entry out of range")
        kk, vv = K[pages, t % page_size], V[pages, t % page_size]  # [n, Hkv, d]
        i = np.arange(lq)[:, None]
        j = np.arange(n)[None, :]
        vis = (j <= i + (n - lq)) if causal else np.ones((lq, n), bool)
        live = vis.any(axis=1)
        for hq in range(Hq):
            s_ = np.where(vis, scale * (Q[qa:qe, hq] @ kk[:, hq // g].T), -np.inf)
            m = np.where(live, s_.max(axis=1), 0.0)
            w = np.where(vis, np.exp(s_ - m[:, None]), 0.0)
            den = np.where(live, w.sum(axis=1), 1.0)
            o[qa:qe, hq] = np.where(live[:, None], (w @ vv[:, hq // g]) / den[:, None], 0.0)
            lse[hq, qa:qe] = np.where(live, m + np.log(den), -np.inf)
    return o, lse
