"""CPU oracle for the attention backward pass -- TEST INFRASTRUCTURE ONLY.

Plain float64 numpy statement of the gradients of exact softmax attention,
written from the definition, with no blocking: for each (batch, query head)
the full score matrix is formed, the softmax taken over the visible keys, and
the gradient of the scalar L = sum(dO * O) with respect to Q, K and V written
out by the chain rule.  Only the tests, the smoke check and the benchmark's
CPU legs may import this module; the CUDA library never does.

Sources followed (page title, section):
  * "Attention Kernel" -- "Backward 与重计算": the backward recomputes the
    local probabilities from Q, K, V, the output and the log-sum-exp, with the
    same softmax scale and mask as the forward and the same GQA head mapping.
    The probabilities themselves are the forward's ("问题与成本"); this module
    forms them directly, which is what the recomputation must reproduce.
  * "Attention 算子加速史" -- FAQ Q1: the backward recomputes the attention
    matrix instead of storing it.

With S = scale * Q K^T + M and P = softmax(S) row by row (rows with no visible
key have P = 0 and O = 0, so they carry no gradient):
    dV = P^T dO                      dP = dO V^T
    dS = P * (dP - rowsum(P * dP))   (the softmax Jacobian applied to dP)
    dQ = scale * dS K                dK = scale * dS^T Q
A KV head shared by g query heads (GQA) receives the sum over those heads.

Pinned in ``tests/test_oracle_bwd_pins.py`` by central finite differences of a
float64 forward through torch's scaled_dot_product_attention, by float64
autograd through that library forward (also with sliding-window, prefix-LM,
block and document masks written element by element in the test), and by
closed forms (equal keys give dQ = 0; the key-sum of dK is 0; the column sums
of dV equal the sums of dO over rows that see a key; the causal first row has
dQ = 0; scale 0).
"""
from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    """bf16 torch tensor, float array or uint16 bf16 bit patterns -> float64 array."""
    if isinstance(x, np.ndarray):
        if x.dtype == np.uint16:
            return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        return x.astype(np.float64)
    return x.detach().cpu().double().numpy()


def visible(Sq: int, Sk: int, klen: int, causal: bool, window: int = 0,
            prefix: int = 0) -> np.ndarray:
    """Boolean [Sq, Sk]: key j is visible to row i iff j < klen and, when causal,
    j <= p with p = i + (klen - Sq) (bottom-right alignment); a sliding window
    w > 0 also requires j > p - w, a prefix P > 0 also admits every j < P
    ("Attention Kernel", section "可编程 mask"; causal only, not both)."""
    i = np.arange(Sq)[:, None]
    j = np.arange(Sk)[None, :]
    vis = j < klen
    if causal:
        p = i + (klen - Sq)
        rule = j <= p
        if window > 0:
            rule = rule & (j > p - window)
        if prefix > 0:
            rule = rule | (j < prefix)
        vis = vis & rule
    elif window > 0 or prefix > 0:
        raise ValueError("window / prefix need the causal mask")
    return vis


def attn_bwd(q, k, v, do, causal, scale, k_lens=None, window=0, prefix=0, block_mask=None):
    """Gradients of L = sum(dO * attn(q, k, v)) in float64.

    q, do [B, Hq, Sq, d]; k, v [B, Hkv, Sk, d] (bf16 tensors, float arrays or
    uint16 bit patterns).  ``k_lens``: optional [B] valid key counts (keys at or
    beyond are masked; the causal diagonal is aligned to the bottom right of
    the first k_lens[b] keys).  ``window`` / ``prefix`` (causal only) and
    ``block_mask`` (uint8 [B, 1 or Hq, ceil(Sq/128), ceil(Sk/128)], 0 hides a
    128 x 128 block) restrict the visible keys as in the forward.  Returns
    (dq, dk, dv) float64 arrays of the input shapes.
    """
    if window > 0 and prefix > 0:
        raise ValueError("window and prefix are exclusive")
    Q, K, V, dO = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Hq, Sq, d = Q.shape
    Bk, Hkv, Sk, dk_ = K.shape
    if K.shape != V.shape or Bk != B or dk_ != d or dO.shape != Q.shape or Hq % Hkv:
        raise ValueError("q/k/v/do shapes disagree")
    g = Hq // Hkv
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    for b in range(B):
        klen = Sk if k_lens is None else int(k_lens[b])
        if not 0 <= klen <= Sk:
            raise ValueError("k_lens out of range")
        vis_b = visible(Sq, Sk, klen, causal, window, prefix)
        for hq in range(Hq):
            kv = hq // g
            vis = vis_b
            if block_mask is not None:
                bm = np.asarray(block_mask)[b, hq if np.asarray(block_mask).shape[1] > 1 else 0]
                vis = vis & np.kron(bm != 0, np.ones((128, 128), bool))[:Sq, :Sk]
            live = vis.any(axis=1)  # rows with at least one visible key
            S = scale * (Q[b, hq] @ K[b, kv].T)
            S = np.where(vis, S, -np.inf)
            m = np.where(live, S.max(axis=1), 0.0)
            E = np.where(vis, np.exp(S - m[:, None]), 0.0)
            den = E.sum(axis=1)
            P = E / np.where(live, den, 1.0)[:, None]
            dP = dO[b, hq] @ V[b, kv].T
            rowdot = (P * dP).sum(axis=1)
            dS = P * (dP - rowdot[:, None])
            dV[b, kv] += P.T @ dO[b, hq]
            dQ[b, hq] = scale * (dS @ K[b, kv])
            dK[b, kv] += scale * (dS.T @ Q[b, hq])
    return dQ, dK, dV


def attn_bwd_varlen(q, k, v, do, cu_seqlens_q, cu_seqlens_k, causal, scale):
    """Gradients for a ragged batch: q, do [total_q, Hq, d], k, v [total_k, Hkv, d]
    packed token-major, cumulative lengths [B + 1]; each sequence is its own
    problem ("Attention Kernel", section "Paged 与 ragged KV"), differentiated
    with ``attn_bwd``.  Returns (dq, dk, dv) float64 of the packed shapes."""
    Q, K, V, dO = _f64(q), _f64(k), _f64(v), _f64(do)
    cq = np.asarray(cu_seqlens_q.cpu().numpy() if hasattr(cu_seqlens_q, "cpu") else cu_seqlens_q)
    ck = np.asarray(cu_seqlens_k.cpu().numpy() if hasattr(cu_seqlens_k, "cpu") else cu_seqlens_k)
    dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    for b in range(len(cq) - 1):
        qa, qb_, ka, kb_ = int(cq[b]), int(cq[b + 1]), int(ck[b]), int(ck[b + 1])
        if qb_ == qa:
            continue
        t = lambda x, a, e: np.ascontiguousarray(x[a:e].transpose(1, 0, 2))[None]
        if kb_ == ka:  # no key: constant zero output, zero gradients
            continue
        gq, gk, gv = attn_bwd(t(Q, qa, qb_), t(K, ka, kb_), t(V, ka, kb_), t(dO, qa, qb_),
                              causal, scale)
        dQ[qa:qb_] = gq[0].transpose(1, 0, 2)
        dK[ka:kb_] = gk[0].transpose(1, 0, 2)
        dV[ka:kb_] = gv[0].transpose(1, 0, 2)
    return dQ, dK, dV
