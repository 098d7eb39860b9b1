"""Seeded synthetic inputs shaped like the notes' workloads.

This module only draws inputs (random numbers, lengths, page placements); it
holds none of the attention arithmetic.  Both the CUDA path and the CPU
oracle are fed the very same bf16 bytes produced here.

Recipe (all on the host, ``torch.Generator().manual_seed(seed)``):
  * Q, K, V: ``randn(float32) * value_scale`` rounded to bf16 (round to nearest
    even), each tensor from its own seed offset so that shapes can change
    without reshuffling the others.
  * Key padding: per sequence, a pad p_b uniform in [0, floor(max_frac * Sk)]
    keys is masked at the end (k_len = Sk - p_b); at least one p_b > 0.
  * Paged decode: seq_lens uniform in [lo, hi]; the cache pool holds exactly
    sum ceil(len/page) pages and a seeded random permutation gives the
    physical page of each logical page; unused block-table slots are -1.
  * Ragged (packed) batches: per-sequence lengths uniform in [lo, hi]; Q, K,
    V drawn packed token-major [total, H, d]; cumulative lengths int32 [B+1].
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

# Seeds fixed per workload: config n uses 1000 + n, the padded variant 1100,
# decode lengths 2000 and the page permutation 2001.
SEED_PADDING = 1100
SEED_DECODE_LENS = 2000
SEED_DECODE_PERM = 2001
SEED_BLOCK_MASK = 211


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    B: int
    Hq: int
    Hkv: int
    S: int
    d: int
    causal: bool
    seed: int
    value_scale: float = 1.0
    padded: bool = False  # per-sequence key padding of 0-25% of Sk

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def flops(self) -> float:
        """4*B*Hq*Sq*Sk*d, halved when causal (the notes' cost model)."""
        f = 4.0 * self.B * self.Hq * self.S * self.S * self.d
        return f / 2 if self.causal else f


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    page_size: int
    len_lo: int
    len_hi: int
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def max_pages_per_seq(self) -> int:
        return -(-self.len_hi // self.page_size)


@dataclass(frozen=True)
class VarlenConfig:
    """A ragged batch: B sequences with len_q = len_k uniform in [len_lo, len_hi]."""
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    causal: bool
    len_lo: int
    len_hi: int
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def lengths(self) -> torch.Tensor:
        g = _gen(self.seed)
        return torch.randint(self.len_lo, self.len_hi + 1, (self.B,), generator=g,
                             dtype=torch.int64).to(torch.int32)

    def flops(self, lengths=None) -> float:
        """sum over sequences of 4*Hq*len^2*d, halved when causal."""
        lens = (self.lengths() if lengths is None else lengths).to(torch.float64)
        f = float(4.0 * self.Hq * self.d * (lens * lens).sum())
        return f / 2 if self.causal else f


@dataclass(frozen=True)
class PagedPrefillConfig:
    """Appending new_tokens query tokens to each of B sequences whose cache already
    holds cached tokens (uniform in [cached_lo, cached_hi]); K/V live in pages."""
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    page_size: int
    new_tokens: int
    cached_lo: int
    cached_hi: int
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def lengths(self):
        """(lens_q, lens_k) int32 [B]: new tokens and cached + new tokens per sequence."""
        g = _gen(self.seed)
        cached = torch.randint(self.cached_lo, self.cached_hi + 1, (self.B,), generator=g,
                               dtype=torch.int64)
        lq = torch.full((self.B,), self.new_tokens, dtype=torch.int64)
        return lq.to(torch.int32), (cached + lq).to(torch.int32)

    def flops(self) -> float:
        """4*Hq*d per visible (query, key) pair; a query at offset i of a sequence
        with len_k keys sees len_k - len_q + i + 1 of them (causal)."""
        lq, lk = (t.to(torch.float64) for t in self.lengths())
        pairs = (lq * (lk - lq) + lq * (lq + 1) / 2).sum()
        return float(4.0 * self.Hq * self.d * pairs)


CONFIGS = {
    "tiny_mha": PrefillConfig("tiny_mha", B=1, Hq=2, Hkv=2, S=256, d=64, causal=False, seed=1001),
    "mha_causal_2k": PrefillConfig("mha_causal_2k", B=4, Hq=16, Hkv=16, S=2048, d=128,
                                   causal=True, seed=1002),
    "gqa_causal_8k": PrefillConfig("gqa_causal_8k", B=2, Hq=32, Hkv=8, S=8192, d=128,
                                   causal=True, seed=1003),
    "gqa_causal_8k_padded": PrefillConfig("gqa_causal_8k_padded", B=2, Hq=32, Hkv=8, S=8192,
                                          d=128, causal=True, seed=1003, padded=True),
    "gqa_causal_32k": PrefillConfig("gqa_causal_32k", B=1, Hq=32, Hkv=8, S=32768, d=128,
                                    causal=True, seed=1004, value_scale=0.5),
    "paged_decode": DecodeConfig("paged_decode", B=64, Hq=32, Hkv=8, d=128, page_size=16,
                                 len_lo=512, len_hi=8192, seed=1005),
    # chunked prefill: 1024 new tokens appended to caches of 0..7168 tokens
    "paged_prefill_gqa": PagedPrefillConfig("paged_prefill_gqa", B=8, Hq=32, Hkv=8, d=128,
                                            page_size=16, new_tokens=1024, cached_lo=0,
                                            cached_hi=7168, seed=1300),
    # the GQA shapes of gqa_causal_8k, as a ragged batch of mixed lengths
    "ragged_gqa_causal": VarlenConfig("ragged_gqa_causal", B=16, Hq=32, Hkv=8, d=128,
                                      causal=True, len_lo=128, len_hi=8192, seed=1200),
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(int(seed))
    return g


def randn_bf16(shape, seed: int, value_scale: float = 1.0) -> torch.Tensor:
    """i.i.d. N(0,1) * value_scale drawn in float32 on the host, rounded to bf16."""
    x = torch.randn(*shape, generator=_gen(seed), dtype=torch.float32)
    if value_scale != 1.0:
        x.mul_(value_scale)
    return x.to(torch.bfloat16)


def prefill_inputs(B, Hq, Hkv, Sq, Sk, d, seed, value_scale=1.0):
    """Q [B,Hq,Sq,d], K and V [B,Hkv,Sk,d] bf16 on the host."""
    q = randn_bf16((B, Hq, Sq, d), seed * 16 + 0, value_scale)
    k = randn_bf16((B, Hkv, Sk, d), seed * 16 + 1, value_scale)
    v = randn_bf16((B, Hkv, Sk, d), seed * 16 + 2, value_scale)
    return q, k, v


def grad_output(B, Hq, Sq, d, seed, value_scale=1.0):
    """dO [B,Hq,Sq,d] bf16 on the host: the gradient a backward pass receives."""
    return randn_bf16((B, Hq, Sq, d), seed * 16 + 3, value_scale)


def block_mask(B: int, heads: int, Sq: int, Sk: int, density: float,
               seed: int = SEED_BLOCK_MASK) -> torch.Tensor:
    """uint8 [B, heads, ceil(Sq/128), ceil(Sk/128)] on the host: each 128 x 128
    (query tile, key tile) block kept (1) with probability ``density``, drawn
    as float32 U[0,1) from a seeded generator."""
    g = torch.Generator().manual_seed(seed)
    return (torch.rand(B, heads, -(-Sq // 128), -(-Sk // 128), generator=g) < density).to(torch.uint8)


def key_padding(B: int, Sk: int, seed: int = SEED_PADDING, max_frac: float = 0.25) -> torch.Tensor:
    """k_lens [B] int32: Sk minus a pad uniform in [0, floor(max_frac*Sk)]; one pad > 0."""
    hi = int(math.floor(max_frac * Sk))
    g = _gen(seed)
    pads = torch.randint(0, hi + 1, (B,), generator=g, dtype=torch.int64)
    if hi > 0 and int(pads.max()) == 0:
        pads[0] = hi
    return (Sk - pads).to(torch.int32)


def config_inputs(cfg: PrefillConfig):
    """(q, k, v, k_lens or None) for a named prefill configuration."""
    q, k, v = prefill_inputs(cfg.B, cfg.Hq, cfg.Hkv, cfg.S, cfg.S, cfg.d, cfg.seed,
                             cfg.value_scale)
    k_lens = key_padding(cfg.B, cfg.S) if cfg.padded else None
    return q, k, v, k_lens


@dataclass
class PagedInputs:
    q: torch.Tensor            # [B, Hq, d] bf16
    k_cache: torch.Tensor      # [num_pages, page_size, Hkv, d] bf16
    v_cache: torch.Tensor      # [num_pages, page_size, Hkv, d] bf16
    block_table: torch.Tensor  # [B, max_pages_per_seq] int32, -1 = unused
    seq_lens: torch.Tensor     # [B] int32
    page_size: int
    extra: dict = field(default_factory=dict)

    @property
    def num_pages(self) -> int:
        return int(self.k_cache.shape[0])


def decode_lengths(B: int, lo: int, hi: int, seed: int = SEED_DECODE_LENS) -> torch.Tensor:
    return torch.randint(lo, hi + 1, (B,), generator=_gen(seed), dtype=torch.int64).to(torch.int32)


def paged_inputs(seq_lens, Hq, Hkv, d, page_size, seed, max_pages_per_seq=None,
                 perm_seed: int = SEED_DECODE_PERM, contiguous: bool = False,
                 extra_pages: int = 0) -> PagedInputs:
    """Paged cache holding exactly the pages the sequences need (+ extra_pages unused).

    Physical page ids come from a seeded random permutation of the pool unless
    ``contiguous`` (logical page i of sequence b then sits right after the
    previous sequence's pages).
    """
    lens = torch.as_tensor(seq_lens, dtype=torch.int32).clone()
    B = lens.shape[0]
    pages_per = [(-(-int(n) // page_size)) for n in lens.tolist()]
    need = sum(pages_per)
    maxp = max_pages_per_seq if max_pages_per_seq is not None else max(pages_per + [1])
    num_pages = need + extra_pages
    if contiguous:
        phys = torch.arange(num_pages, dtype=torch.int64)
    else:
        phys = torch.randperm(num_pages, generator=_gen(perm_seed))
    table = torch.full((B, maxp), -1, dtype=torch.int32)
    pos = 0
    for b, n in enumerate(pages_per):
        if n > maxp:
            raise ValueError("sequence needs more pages than max_pages_per_seq")
        table[b, :n] = phys[pos:pos + n].to(torch.int32)
        pos += n
    q = randn_bf16((B, Hq, d), seed * 16 + 3)
    k_cache = randn_bf16((max(num_pages, 1), page_size, Hkv, d), seed * 16 + 4)
    v_cache = randn_bf16((max(num_pages, 1), page_size, Hkv, d), seed * 16 + 5)
    return PagedInputs(q, k_cache, v_cache, table, lens, page_size)


@dataclass
class PagedFp8Inputs:
    q: torch.Tensor            # [B, Hq, d] bf16
    k_cache: torch.Tensor      # [num_pages, page_size, Hkv, d] uint8 (E4M3 codes)
    v_cache: torch.Tensor      # [num_pages, page_size, Hkv, d] uint8 (E4M3 codes)
    k_scale: torch.Tensor      # [num_pages, Hkv] float32
    v_scale: torch.Tensor      # [num_pages, Hkv] float32
    block_table: torch.Tensor  # [B, max_pages_per_seq] int32, -1 = unused
    seq_lens: torch.Tensor     # [B] int32
    page_size: int

    @property
    def num_pages(self) -> int:
        return int(self.k_cache.shape[0])


E4M3_MAX = 448.0


def quantize_e4m3_per_page(cache: torch.Tensor):
    """bf16 [num_pages, page_size, Hkv, d] -> (E4M3 codes uint8, scales float32
    [num_pages, Hkv]) with scale = amax / 448 per (page, KV head) (1 where the
    block is all zero), the codes being round-to-nearest of x / scale."""
    x = cache.float()
    amax = x.abs().amax(dim=(1, 3))
    sc = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    codes = (x / sc[:, None, :, None]).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), sc.contiguous()


def quantize_e4m3_blocks(x: torch.Tensor, block: int = 128):
    """bf16 [B, H, S, d] -> (E4M3 codes uint8 [B, H, S, d], scales float32
    [B, H, ceil(S / block)]) with scale = amax / 448 per block of `block`
    consecutive rows of one (batch, head) (1 where the block is all zero), the
    codes being round-to-nearest of x / scale (torch's float8_e4m3fn cast)."""
    B, H, S, d = x.shape
    nb = -(-S // block)
    xf = x.float()
    pad = nb * block - S
    if pad:
        xf = torch.cat([xf, torch.zeros(B, H, pad, d)], dim=2)
    blocks = xf.view(B, H, nb, block, d)
    amax = blocks.abs().amax(dim=(3, 4))
    sc = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    codes = (blocks / sc[:, :, :, None, None]).to(torch.float8_e4m3fn).view(torch.uint8)
    codes = codes.view(B, H, nb * block, d)[:, :, :S].contiguous()
    return codes, sc.contiguous()


def fp8_prefill_inputs(B, Hq, Hkv, Sq, Sk, d, seed, value_scale=1.0):
    """Block-scaled E4M3 prefill inputs drawn as ``prefill_inputs`` draws bf16
    ones: (q8, k8, v8, q_scale, k_scale, v_scale)."""
    q, k, v = prefill_inputs(B, Hq, Hkv, Sq, Sk, d, seed, value_scale)
    (q8, qs), (k8, ks), (v8, vs) = (quantize_e4m3_blocks(t) for t in (q, k, v))
    return q8, k8, v8, qs, ks, vs


def fp8_paged_inputs(seq_lens, Hq, Hkv, d, page_size, seed, **kw) -> PagedFp8Inputs:
    """A paged cache as ``paged_inputs`` builds it, quantised to E4M3 with one
    scale per (page, KV head) for K and for V."""
    base = paged_inputs(seq_lens, Hq, Hkv, d, page_size, seed, **kw)
    k8, ks = quantize_e4m3_per_page(base.k_cache)
    v8, vs = quantize_e4m3_per_page(base.v_cache)
    return PagedFp8Inputs(base.q, k8, v8, ks, vs, base.block_table, base.seq_lens, page_size)


def fp8_kv_bytes(seq_lens, Hkv: int, d: int, page_size: int) -> int:
    """Bytes of an FP8 cache the attended tokens occupy: one byte per K and V
    element, plus the K and V scale of every (page, KV head) read."""
    lens = torch.as_tensor(seq_lens, dtype=torch.int64)
    pages = int(((lens + page_size - 1) // page_size).sum())
    return int(lens.sum()) * Hkv * d * 2 + pages * Hkv * 4 * 2


def decode_config_inputs(cfg: DecodeConfig) -> PagedInputs:
    lens = decode_lengths(cfg.B, cfg.len_lo, cfg.len_hi)
    return paged_inputs(lens, cfg.Hq, cfg.Hkv, cfg.d, cfg.page_size, cfg.seed,
                        max_pages_per_seq=cfg.max_pages_per_seq)


def decode_kv_bytes(seq_lens, Hkv: int, d: int, elem_bytes: int = 2) -> int:
    """K+V bytes of the attended tokens: sum(len) * Hkv * d * 2 (K and V)."""
    return int(torch.as_tensor(seq_lens, dtype=torch.int64).sum()) * Hkv * d * elem_bytes * 2


def sample_rows(B, Hq, Sq, n, seed) -> torch.Tensor:
    """n distinct seeded flat row ids (b*Hq + hq)*Sq + i."""
    total = B * Hq * Sq
    n = min(n, total)
    return torch.randperm(total, generator=_gen(seed))[:n].sort().values


def cu_seqlens(lengths) -> torch.Tensor:
    """Cumulative lengths int32 [B+1] (leading 0) of an int tensor or list of lengths."""
    lens = torch.as_tensor(lengths, dtype=torch.int64)
    return torch.cat([torch.zeros(1, dtype=torch.int64), torch.cumsum(lens, 0)]).to(torch.int32)


def varlen_inputs(lens_q, lens_k, Hq: int, Hkv: int, d: int, seed: int, value_scale: float = 1.0):
    """Packed q [sum lens_q, Hq, d], k/v [sum lens_k, Hkv, d] bf16 and cu_seqlens_q/k int32."""
    cu_q, cu_k = cu_seqlens(lens_q), cu_seqlens(lens_k)
    tq, tk = int(cu_q[-1]), int(cu_k[-1])
    q = randn_bf16((tq, Hq, d), seed * 16 + 0, value_scale)
    k = randn_bf16((tk, Hkv, d), seed * 16 + 1, value_scale)
    v = randn_bf16((tk, Hkv, d), seed * 16 + 2, value_scale)
    return q, k, v, cu_q, cu_k


def varlen_config_inputs(cfg: VarlenConfig):
    """(q, k, v, cu_q, cu_k, lengths) for a named ragged configuration."""
    lens = cfg.lengths()
    q, k, v, cu_q, cu_k = varlen_inputs(lens, lens, cfg.Hq, cfg.Hkv, cfg.d, cfg.seed)
    return q, k, v, cu_q, cu_k, lens


def paged_prefill_inputs(lens_q, lens_k, Hq: int, Hkv: int, d: int, page_size: int, seed: int,
                         contiguous: bool = False, max_pages_per_seq=None):
    """(q packed [sum lens_q, Hq, d], cu_seqlens_q, PagedInputs holding the K/V pages,
    block table and seq_lens = lens_k).  The cache is drawn as in ``paged_inputs``."""
    cache = paged_inputs(lens_k, 1, Hkv, d, page_size, seed, max_pages_per_seq=max_pages_per_seq,
                         contiguous=contiguous)
    cu_q = cu_seqlens(lens_q)
    q = randn_bf16((int(cu_q[-1]), Hq, d), seed * 16 + 6)
    return q, cu_q, cache


def paged_prefill_config_inputs(cfg: PagedPrefillConfig):
    lq, lk = cfg.lengths()
    q, cu_q, cache = paged_prefill_inputs(lq, lk, cfg.Hq, cfg.Hkv, cfg.d, cfg.page_size, cfg.seed)
    return q, cu_q, cache, lq, lk
