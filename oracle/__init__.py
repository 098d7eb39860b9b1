"""CPU oracle for exact softmax attention -- TEST INFRASTRUCTURE ONLY.

A plain double-precision C statement of what the attention path computes
(``attn_oracle.c``), loaded through ctypes.  Only the tests, the smoke check
and the benchmark's CPU-baseline / reference legs may import this package; the
product path (the CUDA library and its Python binding) never does, and the
two share no code.

Sources followed (page title, section):
  * "Attention Kernel" -- "问题与成本": O = softmax(QK^T/sqrt(d_h) + M) V with
    Q [B, A, S_q, d_h] and K, V [B, A_kv, S_k, d_h] (GQA).
  * "Attention Kernel" -- "Online softmax" and "Blockwise reference": the
    (m, l, o) merge rule and the zero output for an all -inf row.
  * "Attention Kernel" -- "Paged 与 ragged KV": block = floor(t/q), offset =
    t mod q, physical page through the block table; a ragged batch is a list
    of sequences given by cumulative lengths, each attended on its own.

Every function here is pinned by tests in ``tests/test_oracle_pins.py``
against things other than itself (the notes' worked example evaluated with
``torch.softmax``, closed forms, invariances, ``torch`` SDPA in float64 on
tiny shapes).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

OK = 0
ERR_ARG = 1
ERR_TABLE = 2


def build(force: bool = False) -> str:
    """Compile ``attn_oracle.c`` into ``liboracle.so`` next to it (plain gcc)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c99", "-Wall", "-fPIC", "-shared", "-o", tmp, _SRC,
           "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            D = ctypes.c_double
            L = ctypes.c_int64
            lib.oracle_softmax_attend.argtypes = [P, I, P, I, I, P, P]
            lib.oracle_softmax_attend.restype = I
            lib.oracle_online_attend.argtypes = [P, I, P, I, I, I, P, P, P]
            lib.oracle_online_attend.restype = I
            lib.oracle_attn_fwd_rows.argtypes = [P, P, P, I, I, I, I, I, I, I, D, P, P, L,
                                                 P, P, I]
            lib.oracle_attn_fwd_rows.restype = I
            lib.oracle_attn_fwd_rows_masked.argtypes = [P, P, P, I, I, I, I, I, I, I, D, P, I, I,
                                                        P, L, P, P, I]
            lib.oracle_attn_fwd_rows_masked.restype = I
            lib.oracle_attn_fwd_rows_blocks.argtypes = [P, P, P, I, I, I, I, I, I, I, D, P, I, I,
                                                        P, I, P, L, P, P, I]
            lib.oracle_attn_fwd_rows_blocks.restype = I
            lib.oracle_decode_paged.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, D, P, P, I]
            lib.oracle_decode_paged.restype = I
            _lib = lib
    return _lib


def _threads(n_threads):
    return int(n_threads) if n_threads else (os.cpu_count() or 1)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _bits(x) -> np.ndarray:
    """bf16 tensor (torch) or uint16 array -> contiguous uint16 numpy bit patterns."""
    if isinstance(x, np.ndarray):
        if x.dtype != np.uint16:
            raise TypeError("expected bf16 bit patterns as uint16")
        return np.ascontiguousarray(x)
    import torch
    if x.dtype != torch.bfloat16:
        raise TypeError("expected a bfloat16 tensor")
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy()
                                .view(np.uint16))


class OracleError(RuntimeError):
    def __init__(self, status):
        super().__init__(f"oracle returned status {status}")
        self.status = status


def softmax_attend(scores, values):
    """softmax(scores) @ values for one row, plus its natural-log LSE."""
    s = np.ascontiguousarray(scores, dtype=np.float64)
    v = np.ascontiguousarray(values, dtype=np.float64)
    if s.ndim != 1 or v.ndim != 2:
        raise ValueError("scores must be 1-D and values 2-D")
    o = np.zeros(v.shape[1], np.float64)
    lse = np.zeros(1, np.float64)
    st = _load().oracle_softmax_attend(_ptr(s), s.shape[0], _ptr(v), v.shape[0], v.shape[1],
                                       _ptr(o), _ptr(lse))
    if st != OK:
        raise OracleError(st)
    return o, float(lse[0])


def online_attend(scores, values, block_size, block_order=None):
    """The same row through the blockwise (m, l, o) recurrence."""
    s = np.ascontiguousarray(scores, dtype=np.float64)
    v = np.ascontiguousarray(values, dtype=np.float64)
    if s.ndim != 1 or v.ndim != 2:
        raise ValueError("scores must be 1-D and values 2-D")
    order = None if block_order is None else np.ascontiguousarray(block_order, dtype=np.int32)
    o = np.zeros(v.shape[1], np.float64)
    lse = np.zeros(1, np.float64)
    st = _load().oracle_online_attend(_ptr(s), s.shape[0], _ptr(v), v.shape[0], v.shape[1],
                                      int(block_size), _ptr(order), _ptr(o), _ptr(lse))
    if st != OK:
        raise OracleError(st)
    return o, float(lse[0])


def attn_fwd(q, k, v, causal, scale, k_lens=None, rows=None, n_threads=None, window=0, prefix=0,
             block_mask=None):
    """Exact attention.  q [B,Hq,Sq,d], k/v [B,Hkv,Sk,d] bf16 (torch or uint16 bits).

    ``window`` > 0 (causal only): a row at key position p sees keys (p - window, p];
    ``prefix`` > 0 (causal only): keys below ``prefix`` are visible to every row
    ("Attention Kernel", section "可编程 mask"; not both at once).
    ``block_mask``: optional uint8 [B, 1 or Hq, ceil(Sq/128), ceil(Sk/128)]; a
    zero entry hides every (row, key) pair of that 128 x 128 block.

    ``rows``: optional flat row ids (b*Hq + hq)*Sq + i; default every row.
    Returns (o, lse) as float64 arrays: o [n_rows, d] (or [B,Hq,Sq,d] when
    ``rows`` is None) and lse [n_rows] (or [B,Hq,Sq]).
    """
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, Hq, Sq, d = qb.shape
    Bk, Hkv, Sk, dk = kb.shape
    if kb.shape != vb.shape or Bk != B or dk != d:
        raise ValueError("q/k/v shapes disagree")
    kl = None if k_lens is None else np.ascontiguousarray(np.asarray(k_lens), dtype=np.int32)
    r = None if rows is None else np.ascontiguousarray(np.asarray(rows), dtype=np.int64)
    n = B * Hq * Sq if r is None else r.shape[0]
    o = np.zeros((n, d), np.float64)
    lse = np.zeros(n, np.float64)
    bm, mh = None, 1
    if block_mask is not None:
        bm = np.ascontiguousarray(np.asarray(block_mask), dtype=np.uint8)
        if bm.ndim != 4 or bm.shape[0] != B or bm.shape[1] not in (1, Hq) or \
                bm.shape[2] != -(-Sq // 128) or bm.shape[3] != -(-Sk // 128):
            raise ValueError("block_mask must be uint8 [B, 1 or Hq, ceil(Sq/128), ceil(Sk/128)]")
        mh = bm.shape[1]
    st = _load().oracle_attn_fwd_rows_blocks(_ptr(qb), _ptr(kb), _ptr(vb), B, Hq, Hkv, Sq, Sk, d,
                                             int(bool(causal)), float(scale), _ptr(kl),
                                             int(window), int(prefix), _ptr(bm), mh, _ptr(r), n,
                                             _ptr(o), _ptr(lse), _threads(n_threads))
    if st != OK:
        raise OracleError(st)
    if r is None:
        return o.reshape(B, Hq, Sq, d), lse.reshape(B, Hq, Sq)
    return o, lse


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, causal, scale, n_threads=None,
                    tokens=None):
    """Exact attention over a ragged batch ("Attention Kernel", "Paged 与 ragged KV").

    q [total_q, Hq, d], k/v [total_k, Hkv, d] bf16 (torch or uint16 bits),
    packed; sequence b owns query tokens [cu_q[b], cu_q[b+1]) and key tokens
    [cu_k[b], cu_k[b+1]).  Each sequence is attended on its own, exactly as
    ``attn_fwd`` with B = 1, Sq = len_q, Sk = len_k (bottom-right causal
    diagonal); nothing crosses a sequence boundary.
    Returns (o [total_q, Hq, d], lse [Hq, total_q]) as float64 arrays; rows
    that belong to no sequence stay NaN.  ``tokens``: optional packed query
    token ids; then only those are evaluated (every head) and the result is
    (o [n, Hq, d], lse [Hq, n]) in that order.
    """
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    total_q, Hq, d = qb.shape
    total_k, Hkv, dk = kb.shape
    if kb.shape != vb.shape or dk != d:
        raise ValueError("q/k/v shapes disagree")
    cq = np.asarray(cu_seqlens_q, dtype=np.int64)
    ck = np.asarray(cu_seqlens_k, dtype=np.int64)
    if cq.shape != ck.shape or cq.ndim != 1 or cq.shape[0] < 2:
        raise ValueError("cu_seqlens must both be [B+1]")
    tok = None if tokens is None else np.asarray(tokens, dtype=np.int64)
    n_out = total_q if tok is None else tok.shape[0]
    o = np.full((n_out, Hq, d), np.nan)
    lse = np.full((Hq, n_out), np.nan)
    for b in range(cq.shape[0] - 1):
        q0, q1, k0, k1 = int(cq[b]), int(cq[b + 1]), int(ck[b]), int(ck[b + 1])
        if not (0 <= q0 <= q1 <= total_q and 0 <= k0 <= k1 <= total_k):
            raise ValueError(f"sequence {b}: offsets out of range")
        if q1 == q0:
            continue
        if tok is not None:  # only the requested tokens of this sequence
            sel = np.nonzero((tok >= q0) & (tok < q1))[0]
            if sel.size == 0:
                continue
            qs = np.ascontiguousarray(qb[q0:q1].transpose(1, 0, 2))[None]
            if k1 == k0:
                o[sel] = 0.0
                lse[:, sel] = -np.inf
                continue
            ks = np.ascontiguousarray(kb[k0:k1].transpose(1, 0, 2))[None]
            vs = np.ascontiguousarray(vb[k0:k1].transpose(1, 0, 2))[None]
            n = q1 - q0
            i = tok[sel] - q0
            rows = (np.arange(Hq)[:, None] * n + i[None, :]).reshape(-1)  # head-major
            orow, lrow = attn_fwd(qs, ks, vs, causal, scale, rows=rows, n_threads=n_threads)
            o[sel] = orow.reshape(Hq, sel.size, d).transpose(1, 0, 2)
            lse[:, sel] = lrow.reshape(Hq, sel.size)
            continue
        # [len, H, d] -> [1, H, len, d]
        qs = np.ascontiguousarray(qb[q0:q1].transpose(1, 0, 2))[None]
        if k1 == k0:  # no key: every row is empty
            o[q0:q1] = 0.0
            lse[:, q0:q1] = -np.inf
            continue
        ks = np.ascontiguousarray(kb[k0:k1].transpose(1, 0, 2))[None]
        vs = np.ascontiguousarray(vb[k0:k1].transpose(1, 0, 2))[None]
        ob, lb = attn_fwd(qs, ks, vs, causal, scale, n_threads=n_threads)
        o[q0:q1] = ob[0].transpose(1, 0, 2)
        lse[:, q0:q1] = lb[0]
    return o, lse


def attn_fwd_paged(q, k_cache, v_cache, block_table, cu_seqlens_q, seq_lens_k, causal, scale,
                   n_threads=None, tokens=None):
    """Packed queries over a paged cache ("Attention Kernel", "Paged 与 ragged KV").

    Key token t of sequence b is k_cache[block_table[b][t // page_size], t % page_size]
    (likewise V).  The keys of each sequence are gathered that way and the
    sequence is attended with ``attn_fwd_varlen`` (bottom-right causal
    diagonal: the queries are the last len_q positions).
    Returns (o [total_q, Hq, d], lse [Hq, total_q]) float64; rows of no sequence NaN.
    """
    kc, vc = _bits(k_cache), _bits(v_cache)
    num_pages, page_size, Hkv, d = kc.shape
    tbl = np.asarray(block_table, dtype=np.int64)
    lens = np.asarray(seq_lens_k, dtype=np.int64)
    ks, vs, cu_k = [], [], [0]
    for b in range(lens.shape[0]):
        t = np.arange(int(lens[b]))
        pages = tbl[b, t // page_size]
        if (pages < 0).any() or (pages >= num_pages).any():
            raise OracleError(ERR_TABLE)
        ks.append(kc[pages, t % page_size])
        vs.append(vc[pages, t % page_size])
        cu_k.append(cu_k[-1] + int(lens[b]))
    kp = np.concatenate(ks) if ks else np.zeros((0, Hkv, d), np.uint16)
    vp = np.concatenate(vs) if vs else np.zeros((0, Hkv, d), np.uint16)
    return attn_fwd_varlen(q, kp, vp, cu_seqlens_q, cu_k, causal, scale, n_threads=n_threads,
                           tokens=tokens)


def decode_paged(q, k_cache, v_cache, block_table, seq_lens, scale, n_threads=None):
    """Exact single-query attention over a paged cache.

    q [B,Hq,d]; k_cache/v_cache [num_pages, page_size, Hkv, d] bf16;
    block_table [B, max_pages] int32; seq_lens [B] int32.
    Returns (o [B,Hq,d], lse [B,Hq]) float64.
    """
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    B, Hq, d = qb.shape
    num_pages, page_size, Hkv, dk = kb.shape
    if kb.shape != vb.shape or dk != d:
        raise ValueError("cache shapes disagree")
    tbl = np.ascontiguousarray(np.asarray(block_table), dtype=np.int32)
    lens = np.ascontiguousarray(np.asarray(seq_lens), dtype=np.int32)
    if tbl.ndim != 2 or tbl.shape[0] != B or lens.shape != (B,):
        raise ValueError("block table / seq_lens shapes disagree")
    o = np.zeros((B, Hq, d), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    st = _load().oracle_decode_paged(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(tbl), _ptr(lens), B, Hq,
                                     Hkv, d, page_size, tbl.shape[1], num_pages, float(scale),
                                     _ptr(o), _ptr(lse), _threads(n_threads))
    if st != OK:
        raise OracleError(st)
    return o, lse
