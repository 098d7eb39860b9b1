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

Pinned in ``tests/test_oracle_pins.py`` by central finite differences of the
C forward oracle, by torch autograd in float64 on the explicit formula, and by
closed forms (uniform keys give dQ = 0; the column sums of dV equal the sums
of dO over rows that see a key; the causal first row has dQ = 0).
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


def visible(Sq: int, Sk: int, klen: int, causal: bool) -> np.ndarray:
    """Boolean [Sq, Sk]: key j is visible to row i iff j < klen and, when causal,
    j <= i + (klen - Sq) (bottom-right alignment)."""
    i = np.arange(Sq)[:, None]
    j = np.arange(Sk)[None, :]
    vis = j < klen
    if causal:
        vis = vis & (j <= i + (klen - Sq))
    return vis


def attn_bwd(q, k, v, do, causal, scale, k_lens=None):
    """Gradients of L = sum(dO * attn(q, k, v)) in float64.

    q, do [B, Hq, Sq, d]; k, v [B, Hkv, Sk, d] (bf16 tensors, float arrays or
    uint16 bit patterns).  ``k_lens``: optional [B] valid key counts (keys at or
    beyond are masked; the causal diagonal is aligned to the bottom right of
    the first k_lens[b] keys).  Returns (dq, dk, dv) float64 arrays of the
    input shapes.
    """
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
        vis = visible(Sq, Sk, klen, causal)
        live = vis.any(axis=1)  # rows with at least one visible key
        for hq in range(Hq):
            kv = hq // g
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
