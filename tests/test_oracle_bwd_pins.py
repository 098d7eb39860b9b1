"""Pins for the backward oracle (``oracle/attn_bwd.py``), each against something
other than itself:

* central finite differences of a float64 forward evaluated with torch's
  scaled_dot_product_attention (a library routine), entry by entry;
* torch autograd in float64 through the same library forward, GQA by
  repeating K/V (so the group sum comes from autograd, not from the oracle);
* closed forms and invariants of the softmax Jacobian: equal keys give
  dQ = 0; the key-sum of dK is 0 (softmax is blind to a shift shared by every
  key); the column sums of dV equal the sums of dO over rows that see a key;
  the causal first row has dQ = 0; scale 0 gives dQ = dK = 0 and dV as the
  visible-count-weighted sum of dO; padded keys get no gradient;
* sliding-window, prefix-LM and per-head block masks, and a ragged batch as
  one packed sequence under its document (block-diagonal) mask, against float64
  autograd through SDPA with masks written element by element in the test.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle.attn_bwd import attn_bwd, visible


def _rand(shape, gen, scale=1.0):
    return (torch.randn(shape, generator=gen, dtype=torch.float64) * scale)


def _sdpa_fwd(q, k, v, causal, scale, k_lens):
    """float64 forward through torch SDPA with an explicit boolean mask (rows
    must each see at least one key)."""
    B, Hq, Sq, d = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    g = Hq // Hkv
    kk = k.repeat_interleave(g, dim=1)
    vv = v.repeat_interleave(g, dim=1)
    masks = []
    for b in range(B):
        kl = Sk if k_lens is None else int(k_lens[b])
        masks.append(torch.from_numpy(visible(Sq, Sk, kl, causal)))
    m = torch.stack(masks)[:, None]
    return F.scaled_dot_product_attention(q, kk, vv, attn_mask=m, scale=scale)


CASES = [
    # B, Hq, Hkv, Sq, Sk, d, causal, k_lens
    (1, 2, 1, 5, 7, 4, True, None),
    (2, 2, 2, 6, 6, 3, False, [6, 4]),
    (2, 4, 2, 4, 9, 4, True, [9, 7]),
    (1, 3, 1, 8, 5, 2, False, None),
]


@pytest.mark.parametrize("case", CASES)
def test_bwd_matches_torch_autograd(case):
    B, Hq, Hkv, Sq, Sk, d, causal, k_lens = case
    gen = torch.Generator().manual_seed(11)
    q = _rand((B, Hq, Sq, d), gen).requires_grad_()
    k = _rand((B, Hkv, Sk, d), gen).requires_grad_()
    v = _rand((B, Hkv, Sk, d), gen).requires_grad_()
    do = _rand((B, Hq, Sq, d), gen)
    scale = 0.7
    o = _sdpa_fwd(q, k, v, causal, scale, k_lens)
    (o * do).sum().backward()
    dq, dk, dv = attn_bwd(q.detach(), k.detach(), v.detach(), do, causal, scale, k_lens)
    np.testing.assert_allclose(dq, q.grad.numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(dk, k.grad.numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(dv, v.grad.numpy(), rtol=0, atol=1e-10)


@pytest.mark.parametrize("case", CASES[:3])
def test_bwd_matches_finite_differences(case):
    B, Hq, Hkv, Sq, Sk, d, causal, k_lens = case
    gen = torch.Generator().manual_seed(12)
    q, k, v = _rand((B, Hq, Sq, d), gen), _rand((B, Hkv, Sk, d), gen), _rand((B, Hkv, Sk, d), gen)
    do = _rand((B, Hq, Sq, d), gen)
    scale = 0.6
    dq, dk, dv = attn_bwd(q, k, v, do, causal, scale, k_lens)
    h = 1e-6

    def loss(q_, k_, v_):
        return float((_sdpa_fwd(q_, k_, v_, causal, scale, k_lens) * do).sum())

    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros(x.shape)
        flat = x.view(-1)
        for idx in range(flat.numel()):
            old = float(flat[idx])
            flat[idx] = old + h
            args = {"q": q, "k": k, "v": v}
            lp = loss(args["q"], args["k"], args["v"])
            flat[idx] = old - h
            lm = loss(args["q"], args["k"], args["v"])
            flat[idx] = old
            fd.reshape(-1)[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(grad, fd, rtol=0, atol=2e-7, err_msg=name)


def test_bwd_equal_keys_give_zero_dq_and_keys_sum_of_dk_is_zero():
    gen = torch.Generator().manual_seed(13)
    B, Hq, Hkv, Sq, Sk, d = 1, 2, 1, 6, 6, 4
    q, v, do = _rand((B, Hq, Sq, d), gen), _rand((B, Hkv, Sk, d), gen), _rand((B, Hq, Sq, d), gen)
    k_eq = _rand((1, 1, 1, d), gen).expand(B, Hkv, Sk, d).contiguous()
    dq, _, _ = attn_bwd(q, k_eq, v, do, True, 0.5)
    np.testing.assert_allclose(dq, 0.0, atol=1e-12)
    k = _rand((B, Hkv, Sk, d), gen)
    for causal in (False, True):
        _, dk, _ = attn_bwd(q, k, v, do, causal, 0.5)
        np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)


def test_bwd_dv_column_sums_and_causal_first_row():
    gen = torch.Generator().manual_seed(14)
    B, Hq, Hkv, Sq, Sk, d = 2, 4, 2, 7, 7, 3
    q, k, v = _rand((B, Hq, Sq, d), gen), _rand((B, Hkv, Sk, d), gen), _rand((B, Hkv, Sk, d), gen)
    do = _rand((B, Hq, Sq, d), gen)
    k_lens = [7, 4]
    dq, _, dv = attn_bwd(q, k, v, do, True, 0.8, k_lens)
    # rows i < Sq - k_len see no key under bottom-right causal alignment
    for b in range(B):
        live = np.arange(Sq) >= Sq - k_lens[b]
        for kv in range(Hkv):
            heads = range(kv * 2, kv * 2 + 2)
            want = sum(do[b, h].numpy()[live].sum(axis=0) for h in heads)
            np.testing.assert_allclose(dv[b, kv].sum(axis=0), want, atol=1e-12)
        # the first live row sees exactly one key: P = 1, so dS = 0 and dQ = 0
        np.testing.assert_allclose(dq[b, :, Sq - k_lens[b]], 0.0, atol=1e-12)
        np.testing.assert_allclose(dq[b, :, ~live], 0.0, atol=0)


def test_bwd_scale_zero_closed_form():
    gen = torch.Generator().manual_seed(15)
    B, Hq, Hkv, Sq, Sk, d = 1, 2, 2, 5, 5, 3
    q, k, v = _rand((B, Hq, Sq, d), gen), _rand((B, Hkv, Sk, d), gen), _rand((B, Hkv, Sk, d), gen)
    do = _rand((B, Hq, Sq, d), gen)
    dq, dk, dv = attn_bwd(q, k, v, do, True, 0.0)
    np.testing.assert_allclose(dq, 0.0, atol=0)
    np.testing.assert_allclose(dk, 0.0, atol=0)
    # uniform weights 1/(i+1) over keys 0..i
    w = np.tril(np.ones((Sq, Sk))) / np.arange(1, Sq + 1)[:, None]
    for h in range(Hq):
        np.testing.assert_allclose(dv[0, h], w.T @ do[0, h].numpy(), atol=1e-12)


def test_bwd_gqa_equals_repeated_mha_summed():
    gen = torch.Generator().manual_seed(16)
    B, Hq, Hkv, Sq, Sk, d = 1, 4, 2, 6, 9, 4
    q, k, v = _rand((B, Hq, Sq, d), gen), _rand((B, Hkv, Sk, d), gen), _rand((B, Hkv, Sk, d), gen)
    do = _rand((B, Hq, Sq, d), gen)
    dq, dk, dv = attn_bwd(q, k, v, do, True, 0.4)
    dq2, dk2, dv2 = attn_bwd(q, k.repeat_interleave(2, 1), v.repeat_interleave(2, 1), do, True, 0.4)
    np.testing.assert_allclose(dq, dq2, atol=1e-12)
    np.testing.assert_allclose(dk, dk2.reshape(B, Hkv, 2, Sk, d).sum(axis=2), atol=1e-12)
    np.testing.assert_allclose(dv, dv2.reshape(B, Hkv, 2, Sk, d).sum(axis=2), atol=1e-12)


def test_bwd_padded_keys_get_no_gradient_and_noncausal_padding_is_truncation():
    gen = torch.Generator().manual_seed(17)
    B, Hq, Hkv, Sq, Sk, d = 1, 2, 1, 5, 8, 3
    q, k, v = _rand((B, Hq, Sq, d), gen), _rand((B, Hkv, Sk, d), gen), _rand((B, Hkv, Sk, d), gen)
    do = _rand((B, Hq, Sq, d), gen)
    dq, dk, dv = attn_bwd(q, k, v, do, False, 0.5, k_lens=[5])
    np.testing.assert_allclose(dk[:, :, 5:], 0.0, atol=0)
    np.testing.assert_allclose(dv[:, :, 5:], 0.0, atol=0)
    dq2, dk2, dv2 = attn_bwd(q, k[:, :, :5], v[:, :, :5], do, False, 0.5)
    np.testing.assert_allclose(dq, dq2, atol=1e-12)
    np.testing.assert_allclose(dk[:, :, :5], dk2, atol=1e-12)
    np.testing.assert_allclose(dv[:, :, :5], dv2, atol=1e-12)
    # every key masked: nothing flows anywhere
    dq0, dk0, dv0 = attn_bwd(q, k, v, do, True, 0.5, k_lens=[0])
    assert not dq0.any() and not dk0.any() and not dv0.any()


def test_bwd_accepts_bf16_bits():
    gen = torch.Generator().manual_seed(18)
    q = torch.randn((1, 1, 3, 2), generator=gen).to(torch.bfloat16)
    k = torch.randn((1, 1, 3, 2), generator=gen).to(torch.bfloat16)
    v = torch.randn((1, 1, 3, 2), generator=gen).to(torch.bfloat16)
    do = torch.randn((1, 1, 3, 2), generator=gen).to(torch.bfloat16)
    bits = [x.view(torch.int16).numpy().view(np.uint16) for x in (q, k, v, do)]
    a = attn_bwd(q, k, v, do, True, 0.5)
    b = attn_bwd(*bits, True, 0.5)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


# --------------------------------------------------------------------------- masks and ragged batches

from oracle.attn_bwd import attn_bwd_varlen  # noqa: E402


def _sdpa_masked(q, k, v, scale, mask):
    """float64 SDPA with an explicit boolean mask [B or 1, Hq or 1, Sq, Sk] (GQA by
    repeating K/V); every row must see a key."""
    g = q.shape[1] // k.shape[1]
    return F.scaled_dot_product_attention(q, k.repeat_interleave(g, 1), v.repeat_interleave(g, 1),
                                          attn_mask=mask, scale=scale)


def _rule_mask(Sq, Sk, window=0, prefix=0, block=None):
    """The causal visibility rule written element by element (independently of
    the oracle's vectorised form): row i sits at key position p = i + Sk - Sq
    and sees key j iff j <= p and, with a window w, p - j < w; with a prefix P,
    also every j < P; a block mask entry 0 hides (i // 128, j // 128)."""
    m = torch.zeros((Sq, Sk), dtype=torch.bool)
    for i in range(Sq):
        p = i + Sk - Sq
        for j in range(Sk):
            ok = j <= p and (window == 0 or p - j < window)
            if prefix > 0 and j < prefix:
                ok = True
            if block is not None and not block[i // 128][j // 128]:
                ok = False
            m[i, j] = ok
    return m


def _grads_autograd(q, k, v, do, scale, mask):
    q, k, v = (x.clone().requires_grad_() for x in (q, k, v))
    (_sdpa_masked(q, k, v, scale, mask) * do).sum().backward()
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("Sq,Sk,window,prefix", [(9, 9, 3, 0), (6, 11, 4, 0), (10, 10, 0, 3),
                                                   (7, 12, 0, 8)])
def test_bwd_window_and_prefix_match_autograd(Sq, Sk, window, prefix):
    gen = torch.Generator().manual_seed(19)
    B, Hq, Hkv, d = 1, 4, 2, 3
    q, k, v = _rand((B, Hq, Sq, d), gen), _rand((B, Hkv, Sk, d), gen), _rand((B, Hkv, Sk, d), gen)
    do = _rand((B, Hq, Sq, d), gen)
    mask = _rule_mask(Sq, Sk, window, prefix)[None, None]
    ref = _grads_autograd(q, k, v, do, 0.6, mask)
    got = attn_bwd(q, k, v, do, True, 0.6, window=window, prefix=prefix)
    for x, y in zip(got, ref):
        np.testing.assert_allclose(x, y, rtol=0, atol=1e-10)


def test_bwd_block_mask_matches_autograd():
    """A per-head 128 x 128 block mask on 300 x 300 causal problems (every row
    keeps its diagonal block, so each row sees a key)."""
    gen = torch.Generator().manual_seed(20)
    B, Hq, Hkv, S, d = 1, 2, 1, 300, 4
    q, k, v = _rand((B, Hq, S, d), gen), _rand((B, Hkv, S, d), gen), _rand((B, Hkv, S, d), gen)
    do = _rand((B, Hq, S, d), gen)
    bm = np.ones((B, Hq, 3, 3), np.uint8)
    bm[0, 0, 2, 0] = 0
    bm[0, 1, 1, 0] = 0
    bm[0, 1, 2, 1] = 0
    mask = torch.stack([_rule_mask(S, S, block=bm[0, h]) for h in range(Hq)])
    ref = _grads_autograd(q, k, v, do, 0.5, mask[None])
    got = attn_bwd(q, k, v, do, True, 0.5, block_mask=bm)
    for x, y in zip(got, ref):
        np.testing.assert_allclose(x, y, rtol=0, atol=1e-10)
    # an all-ones mask is no mask
    ones = attn_bwd(q, k, v, do, True, 0.5, block_mask=np.ones_like(bm))
    plain = attn_bwd(q, k, v, do, True, 0.5)
    for x, y in zip(ones, plain):
        np.testing.assert_array_equal(x, y)


def test_bwd_ragged_batch_is_the_document_masked_packed_sequence():
    """A ragged batch differentiated per sequence equals autograd of one packed
    sequence under the block-diagonal (document) mask with bottom-right causal
    alignment inside each document."""
    gen = torch.Generator().manual_seed(21)
    lq, lk = [3, 5, 2], [3, 7, 4]
    Hq, Hkv, d = 2, 1, 3
    cq = np.concatenate([[0], np.cumsum(lq)])
    ck = np.concatenate([[0], np.cumsum(lk)])
    q, do = _rand((cq[-1], Hq, d), gen), _rand((cq[-1], Hq, d), gen)
    k, v = _rand((ck[-1], Hkv, d), gen), _rand((ck[-1], Hkv, d), gen)
    got = attn_bwd_varlen(q, k, v, do, cq, ck, True, 0.7)
    mask = np.zeros((cq[-1], ck[-1]), bool)
    for b in range(len(lq)):
        mask[cq[b]:cq[b + 1], ck[b]:ck[b + 1]] = _rule_mask(lq[b], lk[b]).numpy()
    pk = lambda x: x.permute(1, 0, 2)[None]  # packed [T, H, d] -> [1, H, T, d]
    ref = _grads_autograd(pk(q), pk(k), pk(v), pk(do), 0.7, torch.from_numpy(mask)[None, None])
    for x, y in zip(got, ref):
        np.testing.assert_allclose(x, y[0].transpose(1, 0, 2), rtol=0, atol=1e-10)
    # a sequence with no keys contributes nothing and receives nothing
    ck2 = ck.copy()
    ck2[1:] = ck[1:] - ck[1]  # sequence 0 keeps 0 keys; the others shift down
    g0 = attn_bwd_varlen(q, k[:ck2[-1]], v[:ck2[-1]], do, cq, ck2, True, 0.7)
    assert not g0[0][:cq[1]].any()
